// Forward of causal packed-document attention, MXFP8 path, for sm_100a
// (FLAMIA page, sec. "FLAMIA Mimarisi ve Temel Tasarim Ilkeleri": MXFP8
// operands with shared E8M0 scales, token-block scaling, leak guards,
// document-local scales; GPT page secs. 3-6 for the attention itself).
//
// Fused quantisation: Q is quantised on load by this kernel (each query tile
// is read by exactly one work item), per token for the scores, and written to
// ctx in both forms for the backward; K and V, which every later query tile
// of the document streams again, come from a prepass in token-block form (one
// scale per 32 tokens x 32 channels) and per-token form (one scale per token x
// 32 channels), and the diagonal tile's per-token V is dequantised on load for
// its exact bf16 product.  Leak guard (rule L): a query of 32-token block b
// sees keys of earlier blocks through the token-block forms and keys of its
// own block through the per-token forms, so no shared scale pools a future
// token.
//
// One persistent CTA per SM, 576 threads; work item = (document, 128-row
// query tile, head).  Warps 0-15: one thread per (query row, 32-key block):
// warpgroup wg takes key block wg of every tile, i.e. one MX scale block of
// P~ (softmax, P quantisation, epilogue of O columns [32 wg, 32 wg + 32));
// the four threads of a row exchange their block maxima through shared
// memory (an mbarrier per row quarter, bounded waits) so they all move the
// reference M alike, and add their partial row sums at the end.  At the start
// of an item the same threads, as (query row, 32-channel group), quantise the
// item's Q and dequantise its diagonal V.  Warp 16: loads (TMA for K and V
// codes, plain loads for their scale bytes, staged into the 512-byte blocks
// tcgen05.cp copies to TMEM); warp 17 (one lane): MMAs.
//  * S = Q K^T for every key tile: block-scaled FP8 MMA (kind::mxf8f6f4,
//    E8M0 scales in TMEM) with K in token-block form; on the diagonal tile a
//    second S with K per token, selected on the diagonal 32x32 blocks.
//  * P: u = 2^(S log2 e - M) with an integer running reference M (moved only
//    when the row maximum grows by more than 8), quantised per (row, 32-key
//    block) to E4M3 with an E8M0 scale.  MX quantisation is invariant under
//    powers of two, so every M yields the same codes as the final one.
//  * O += P~ V~: block-scaled FP8 MMA with V in token-block form (MN-major);
//    on the diagonal tile the diagonal 32x32 blocks of P~ are taken out of the
//    FP8 operand and multiplied exactly with the dequantised per-token V in a
//    bf16 MMA (per-token V scales vary along the contraction, which an MX
//    block scale cannot express).
// TMEM: S buffers [0,128) and [128,256) (the diagonal tile's per-token S uses
// the buffer the previous tile freed), O [256,384), scale factors from 384.
//
// Mixed NVFP4/FP8 path (kNv): the scores take Q and K in NVFP4 (E2M1 codes,
// one E4M3 scale per 16 channels of one token, kind::mxf4nvf4 MMAs, two per
// tile with K = 64); Q is quantised on load to NVFP4 (its token-block MXFP8
// form and its NVFP4 form go to ctx for the backward), K's NVFP4 tiles come
// from the prepass.  NVFP4 blocks lie inside one token, so the diagonal
// tile's second S (the "per-token" one) is the same product on the diagonal
// key tile and the softmax warps run unchanged; P~ V is the MXFP8 path's.
#include <cuda_bf16.h>

#include "internal.h"
#include "mx.cuh"
#include "nv.cuh"
#include "ptx.cuh"
#include "sched.cuh"

namespace fapk {

namespace {

constexpr int kThreads = 576;
constexpr int kLoadWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kComputeWarps = 16;
constexpr int kSlots = 6;
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;

// shared memory plan (bytes, 1024-aligned tiles)
constexpr int kCodeTile = 128 * 128;      // 128 rows x 128 fp8 codes
constexpr int kBf16Tile = 128 * 128 * 2;  // 128 rows x 128 bf16
constexpr int kBox = 128 * 64 * 2;        // one 64-channel bf16 box
constexpr int oQ = 0;
constexpr int oKpt = oQ + kCodeTile;
constexpr int oVpt = oKpt + kCodeTile;
constexpr int oP = oVpt + kBf16Tile;
constexpr int oPd = oP + kCodeTile;
constexpr int oRing = oPd + kBf16Tile;
constexpr int oSf = oRing + kSlots * kCodeTile;  // sfQ, sfKpt, sfP, sfRing[kSlots]
constexpr int kSfBlk = 512;
// mixed path: the second scale block (channels 64..127) of sfQ, sfKpt, sfRing[kSlots]
constexpr int oSf2 = oSf + (3 + kSlots) * kSfBlk;
constexpr int oXmax = oSf2 + (2 + kSlots) * kSfBlk;  // block maxima [2][4][128] (by tile parity)
constexpr int oLsum = oXmax + 2 * 4 * 128 * 4;       // partial row sums [4][128]
constexpr int oBars = oLsum + 4 * 128 * 4;
// q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full, pv_done, o_full, o_free, fin,
// one row-exchange barrier per row quarter, kpt_full, vd_full, the unit ring's full[8] and empty[8]
constexpr int kNumBars = 2 + 2 * kSlots + 13 + 2 * kUnitRing;
constexpr int kSmemBytes = oBars + kNumBars * 8 + 16 + kUnitRingBytes + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory exceeds the 227 KB a CTA may use");

// TMEM columns
constexpr uint32_t kS0 = 0, kS1 = 128, kO = 256;
constexpr uint32_t kSfQ = 384, kSfK = 388, kSfKpt = 392, kSfP = 396, kSfV = 400;
constexpr uint32_t kSfQ2 = 404, kSfK2 = 408, kSfKpt2 = 412;  // mixed path: channels 64..127
// the K scale columns of odd tiles: the copy for S(j + 2) is issued before
// S(j + 1), which reads the other set, has been seen complete, so it must not
// overwrite that set (it overwrites S(j)'s, which the softmax warps have read)
constexpr uint32_t kSfK1 = 416, kSfK21 = 420;
constexpr uint32_t kSfCols[] = {kSfQ, kSfK, kSfKpt, kSfP, kSfV, kSfQ2, kSfK2, kSfKpt2, kSfK1, kSfK21};
static_assert(sf_cols_ok(kSfCols, kO + 128), "forward TMEM scale columns overlap");
constexpr int kNvTile = 128 * 64;  // 128 rows x 128 E2M1 codes

struct Params {
  const int32_t* cu;
  SchedView sched;
  const __nv_bfloat16* q;  // Q [T][Hq][128] (bf16 input, quantised on load)
  uint8_t* q_vpt;          // out: Q per-token codes [T][Hq][128] (ctx); null: no saved state
                           // for a backward (then q_spt.. and o_resid are not written either)
  uint8_t* q_spt;          // out: Q per-token scales [T][Hq][4]
  uint8_t* q_vtb;          // out: Q token-block codes [T][Hq][128]
  uint8_t* q_stb;          // out: Q token-block scales [slots][Hq][4]
  const uint8_t* v_vpt;    // V per-token codes [T][Hkv][128] (diagonal tile)
  const uint8_t* v_spt;    // V per-token scales [T][Hkv][4]
  const uint8_t* k_stb;   // K token-block scales [slots][Hkv][4]
  const uint8_t* k_spt;   // K per-token scales [T][Hkv][4]
  const uint8_t* v_stb;   // V token-block scales [slots][Hkv][4]
  // mixed path
  const uint8_t* k_nvs;   // K NVFP4 scales [T][Hkv][8]
  uint8_t* q_nvv;         // out: Q NVFP4 codes [T][Hq][64] (ctx); null: no saved state
  uint8_t* q_nvs;         // out: Q NVFP4 scales [T][Hq][8]
  float nv_g_q, nv_six_g_q;  // Q's decode scale g and fp32(6 g)
  __nv_bfloat16* o;
  float* lse;
  __nv_bfloat16* o_resid;
  DeviceStatus* status;
  uint64_t timeout_ns;
  int T, Hq, Hkv, n_docs;
  int d;  // head dimension of Q and O (64 or 128); the codes always have 128 per row
  float scale_log2;
  int rule;
  int wide;  // O and its residual 32-byte aligned: 32-byte stores
  unsigned long long* cta_times;  // per-CTA (start, end) records, or null
};

struct Item {
  int doc, s, e, h, g, q0, m, n;  // query tile m; n = m + 1 key tiles, tile n-1 is the diagonal
};

__device__ __forceinline__ Item decode(const Params& p, const UnitInfo& un) {
  Item it;
  const int m = un.tile;
  it.doc = un.doc;
  it.h = un.h;
  it.g = it.h / (p.Hq / p.Hkv);
  it.s = un.s;
  it.e = un.e;
  it.q0 = it.s + 128 * m;
  it.m = m;
  it.n = m + 1;
  return it;
}

// Per item, one thread per (row, 32-channel group wg) of its 128 rows (tokens
// q0 + row; rows past the document end are zeros and are not stored):
//  * stage_q: Q quantised per token into the MMA operand sQ (K-major FP8,
//    128-byte swizzle) and its scale block sfQ, and, for the backward, into
//    ctx in per-token and token-block form (the warp's 32 rows are one
//    document-local token block, since tiles start at the document start);
//  * stage_v: the diagonal tile's per-token V (its keys are the same tokens)
//    dequantised to bf16 into sVpt (two 64-channel boxes, 128-byte swizzle);
//  * prefetch: the item's Q row and diagonal V codes into L2, ahead of both.
__device__ __forceinline__ void prefetch_item(const Params& p, const Item& it, int row, int wg) {
  const int t = it.q0 + row;
  if (t >= it.e) return;
  const __nv_bfloat16* q = p.q + ((size_t)t * p.Hq + it.h) * 128 + 32 * wg;
  const uint8_t* v = p.v_vpt + ((size_t)t * p.Hkv + it.g) * 128 + 32 * wg;
  asm volatile("prefetch.global.L2 [%0];" ::"l"(q));
  asm volatile("prefetch.global.L2 [%0];" ::"l"(v));
}

template <bool kNv>
__device__ __forceinline__ void stage_q(const Params& p, const Item& it, int row, int wg, uint8_t* sQ,
                                        uint8_t* sfQ) {
  const int t = it.q0 + row;
  const bool in_doc = t < it.e;
  float f[32];
  if (in_doc && 32 * wg < p.d) {  // channels past d (d = 64) are zeros
    const uint4* src = reinterpret_cast<const uint4*>(p.q + ((size_t)t * p.Hq + it.h) * p.d + 32 * wg);
    uint4 raw[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) raw[c] = __ldg(src + c);
#pragma unroll
    for (int c = 0; c < 4; ++c) unpack8(raw[c], *reinterpret_cast<float(*)[8]>(&f[8 * c]));
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) f[c] = 0.f;
  }
  float a = 0.f;
#pragma unroll
  for (int c = 0; c < 32; ++c) a = fmaxf(a, fabsf(f[c]));
  uint2 cw[4];
  if constexpr (kNv) {
    // NVFP4 for the scores: channels 32 wg .. 32 wg + 31 are two 16-channel
    // blocks, 16 bytes of codes = chunk wg of the 64-byte row; their scale
    // bytes 2 wg, 2 wg + 1 go to the word of MMA k-step wg >> 1
    uint32_t c0[2], c1[2];
    const uint32_t s0 = nv_quant16(&f[0], p.nv_six_g_q, p.nv_g_q, c0);
    const uint32_t s1 = nv_quant16(&f[16], p.nv_six_g_q, p.nv_g_q, c1);
    const uint4 codes = make_uint4(c0[0], c0[1], c1[0], c1[1]);
    *reinterpret_cast<uint4*>(sQ + sw64_chunk(row, wg)) = codes;
    const uint16_t sw = (uint16_t)(s0 | (s1 << 8));
    *reinterpret_cast<uint16_t*>(sfQ + (wg >> 1) * (oSf2 - oSf) + (row & 31) * 16 + (row >> 5) * 4 + 2 * (wg & 1)) = sw;
    if (!p.q_nvv) return;  // inference: Q's forms are not kept
    if (in_doc) {
      *reinterpret_cast<uint4*>(p.q_nvv + ((size_t)t * p.Hq + it.h) * 64 + 16 * wg) = codes;
      *reinterpret_cast<uint16_t*>(p.q_nvs + ((size_t)t * p.Hq + it.h) * 8 + 2 * wg) = sw;
    }
  } else {
    // per-token form
    const int X = mx_block_exponent(a, p.rule);
#pragma unroll
    for (int c = 0; c < 4; ++c) cw[c] = encode8(*reinterpret_cast<const float(*)[8]>(&f[8 * c]), X);
    uint8_t* prow = sQ + row * 128;
    *reinterpret_cast<uint4*>(prow + (((2 * wg) ^ (row & 7)) << 4)) = make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
    *reinterpret_cast<uint4*>(prow + (((2 * wg + 1) ^ (row & 7)) << 4)) = make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
    sfQ[(row & 31) * 16 + (row >> 5) * 4 + wg] = (uint8_t)(X + 127);
    if (!p.q_vpt) return;  // inference: Q's forms are not kept
    if (in_doc) {
      uint4* dst = reinterpret_cast<uint4*>(p.q_vpt + ((size_t)t * p.Hq + it.h) * 128 + 32 * wg);
      dst[0] = make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
      dst[1] = make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
      p.q_spt[((size_t)t * p.Hq + it.h) * 4 + wg] = (uint8_t)(X + 127);
    }
  }
  const size_t qo = ((size_t)t * p.Hq + it.h) * 128 + 32 * wg;
  // token-block form: the warp's 32 rows, this channel group
  float atb = a;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) atb = fmaxf(atb, __shfl_xor_sync(0xFFFFFFFFu, atb, off));
  const int Xtb = mx_block_exponent(atb, p.rule);
#pragma unroll
  for (int c = 0; c < 4; ++c) cw[c] = encode8(*reinterpret_cast<const float(*)[8]>(&f[8 * c]), Xtb);
  if (in_doc) {
    uint4* dst = reinterpret_cast<uint4*>(p.q_vtb + qo);
    dst[0] = make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
    dst[1] = make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
  }
  const int quarter = row >> 5;
  if ((row & 31) == 0 && it.q0 + 32 * quarter < it.e) {
    const size_t slot = (size_t)(it.s >> 5) + it.doc + 4 * it.m + quarter;
    p.q_stb[(slot * p.Hq + it.h) * 4 + wg] = (uint8_t)(Xtb + 127);
  }
}

__device__ __forceinline__ void stage_v(const Params& p, const Item& it, int row, int wg, uint8_t* sVpt) {
  const int t = it.q0 + row;
  uint4 vc[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
  uint32_t vs = 127u;
  if (t < it.e) {
    const uint4* vsrc = reinterpret_cast<const uint4*>(p.v_vpt + ((size_t)t * p.Hkv + it.g) * 128 + 32 * wg);
    vc[0] = __ldg(vsrc);
    vc[1] = __ldg(vsrc + 1);
    vs = __ldg(p.v_spt + ((size_t)t * p.Hkv + it.g) * 4 + wg);
  }
  // per-token codes -> bf16 (exact), channels 32 wg .. 32 wg + 31
  const int Xv = (int)vs - 127;
  const uint4 d0 = dequant8_bf16(make_uint2(vc[0].x, vc[0].y), Xv);
  const uint4 d1 = dequant8_bf16(make_uint2(vc[0].z, vc[0].w), Xv);
  const uint4 d2 = dequant8_bf16(make_uint2(vc[1].x, vc[1].y), Xv);
  const uint4 d3 = dequant8_bf16(make_uint2(vc[1].z, vc[1].w), Xv);
  uint8_t* vrow = sVpt + (wg >> 1) * kBox + row * 128;
  const int c0 = (wg & 1) * 4;
  *reinterpret_cast<uint4*>(vrow + (((c0 + 0) ^ (row & 7)) << 4)) = d0;
  *reinterpret_cast<uint4*>(vrow + (((c0 + 1) ^ (row & 7)) << 4)) = d1;
  *reinterpret_cast<uint4*>(vrow + (((c0 + 2) ^ (row & 7)) << 4)) = d2;
  *reinterpret_cast<uint4*>(vrow + (((c0 + 3) ^ (row & 7)) << 4)) = d3;
}

// tm_ktb, tm_kpt: K's token-block and per-token MXFP8 codes, or (kNv) both
// K's NVFP4 codes
template <bool kNv>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_mxfp8_kernel(const __grid_constant__ CUtensorMap tm_ktb, const __grid_constant__ CUtensorMap tm_kpt,
                     const __grid_constant__ CUtensorMap tm_vtb, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + oQ;
  uint8_t* sKpt = smem + oKpt;
  uint8_t* sVpt = smem + oVpt;
  uint8_t* sP = smem + oP;
  uint8_t* sPd = smem + oPd;
  uint8_t* sRing = smem + oRing;
  uint8_t* sfQ = smem + oSf;
  uint8_t* sfKpt = sfQ + kSfBlk;
  uint8_t* sfP = sfQ + 2 * kSfBlk;
  uint8_t* sfRing = sfQ + 3 * kSfBlk;
  uint8_t* sfKpt2 = smem + oSf2 + kSfBlk;   // mixed path: second scale blocks
  uint8_t* sfRing2 = smem + oSf2 + 2 * kSfBlk;
  constexpr uint32_t kKBytes = kNv ? kNvTile : kCodeTile;  // bytes of one K tile
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + oBars);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = bars + 2 + kSlots;
  // one "scores ready" barrier per S buffer: tile j signals s_full[j & 1], so
  // no barrier ever runs more than one phase ahead of its waiters
  uint64_t* s_full = bars + 2 + 2 * kSlots;  // [2]
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = s_full + 3;
  uint64_t* o_full = s_full + 4;
  uint64_t* o_free = s_full + 5;
  uint64_t* fin = s_full + 6;
  uint64_t* xbar = s_full + 7;  // [4]
  uint64_t* kpt_full = s_full + 11;  // the diagonal per-token K and its scales (loader)
  uint64_t* vd_full = s_full + 12;   // the diagonal V dequantised to bf16 (compute warps)
  const UnitRing ring{reinterpret_cast<int*>(bars + kNumBars) + 4, bars + kNumBars - 2 * kUnitRing,
                      bars + kNumBars - kUnitRing};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, kComputeWarps);  // Q staged by the compute warps
    mbar_init(kpt_full, 32);
    mbar_init(vd_full, kComputeWarps);
    mbar_init(q_empty, 1);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(kv_full + i, 32);
      mbar_init(kv_empty + i, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_full + 1, 1);
    mbar_init(p_full, kComputeWarps);
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, kComputeWarps);
    mbar_init(fin, 1);
    unit_ring_init(ring, 1 + kComputeWarps);  // the MMA thread and the softmax warps
    for (int i = 0; i < 4; ++i) mbar_init(xbar + i, 4);
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
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) {  // scheduler balance record
    if (blockIdx.x == 0) p.cta_times[0] = gridDim.x;
    p.cta_times[1 + 2 * blockIdx.x] = globaltimer_ns();
  }
  const Watchdog wd{p.status, abort_flag, p.timeout_ns};
  const UnitSpace us = unit_space(p.sched, p.Hq, kSchedQ);
  const int n_units = us.n_units();

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ loads
    uint32_t kv_it = 0, kpt_loads = 0;
    int unit_i = 0;
    bool ok = true;
    for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
      const UnitInfo un = unit_produce_warp(ring, us, p.cu, p.sched.next, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      const Item it = decode(p, un);
      for (int j = 0; j < it.n && ok; ++j) {
        for (int kv = 0; kv < 2; ++kv, ++kv_it) {
          const int slot = kv_it % kSlots;
          const uint32_t use = kv_it / kSlots;
          // the scale words' global reads first, so that their latency overlaps the wait
          uint4 wsf, wsf2 = make_uint4(0u, 0u, 0u, 0u);
          if (kNv && kv == 0) {
            // K rows = keys: the NVFP4 scale words (channels 0..63, 64..127) of each key
            const int k0 = it.s + 128 * j;
            const uint2 w0 = nv_scale_words(p.k_nvs, k0 + lane, p.T, p.Hkv, it.g);
            const uint2 w1 = nv_scale_words(p.k_nvs, k0 + lane + 32, p.T, p.Hkv, it.g);
            const uint2 w2 = nv_scale_words(p.k_nvs, k0 + lane + 64, p.T, p.Hkv, it.g);
            const uint2 w3 = nv_scale_words(p.k_nvs, k0 + lane + 96, p.T, p.Hkv, it.g);
            wsf = make_uint4(w0.x, w1.x, w2.x, w3.x);
            wsf2 = make_uint4(w0.y, w1.y, w2.y, w3.y);
          } else if (kv == 0) {
            // K rows = keys: the scale word of the key's token block
            wsf.x = tb_word(p.k_stb, it.s, it.e, it.doc, 4 * j + 0, p.Hkv, it.g);
            wsf.y = tb_word(p.k_stb, it.s, it.e, it.doc, 4 * j + 1, p.Hkv, it.g);
            wsf.z = tb_word(p.k_stb, it.s, it.e, it.doc, 4 * j + 2, p.Hkv, it.g);
            wsf.w = tb_word(p.k_stb, it.s, it.e, it.doc, 4 * j + 3, p.Hkv, it.g);
          } else {
            // V as B of P V: rows = channels c = lane + 32 r1 (group r1), K
            // blocks = the tile's 4 key blocks; byte kb of word r1 is the
            // token-block scale of (key block 4j + kb, channel group r1)
            uint32_t wv[4] = {0, 0, 0, 0};
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint32_t t = tb_word(p.v_stb, it.s, it.e, it.doc, 4 * j + kb, p.Hkv, it.g);
#pragma unroll
              for (int r1 = 0; r1 < 4; ++r1) wv[r1] |= ((t >> (8 * r1)) & 0xFFu) << (8 * kb);
            }
            wsf = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
          if (use > 0 && !warp_wait(kv_empty + slot, (use - 1) & 1, wd, 52)) { ok = false; break; }
          if (kNv && kv == 0) reinterpret_cast<uint4*>(sfRing2 + slot * kSfBlk)[lane] = wsf2;
          reinterpret_cast<uint4*>(sfRing + slot * kSfBlk)[lane] = wsf;
          fence_proxy_async_smem();
          if (lane == 0) {
            mbar_arrive_expect_tx(kv_full + slot, kv ? kCodeTile : kKBytes);
            tma_load_3d(sRing + slot * kCodeTile, kv ? &tm_vtb : &tm_ktb, kv_full + slot, 0, it.g, it.s + 128 * j);
          } else {
            mbar_arrive(kv_full + slot);
          }
        }
        if (j == it.n - 1 && ok) {
          // the diagonal per-token K and its scale block (row r = lane + 32 r1
          // -> bytes 16 lane + 4 r1 .. +3), once every MMA of the previous
          // item has read the previous ones; after the item's last K and V
          // (the per-token scores come last), so that the item's streamed
          // tiles never wait for the previous item to finish
          uint4 wk, wk2 = make_uint4(0u, 0u, 0u, 0u);
          if constexpr (kNv) {
            // the diagonal key tile's NVFP4 codes and scales (the same scores
            // as the ring's copy of that tile)
            const uint2 w0 = nv_scale_words(p.k_nvs, it.q0 + lane, p.T, p.Hkv, it.g);
            const uint2 w1 = nv_scale_words(p.k_nvs, it.q0 + lane + 32, p.T, p.Hkv, it.g);
            const uint2 w2 = nv_scale_words(p.k_nvs, it.q0 + lane + 64, p.T, p.Hkv, it.g);
            const uint2 w3 = nv_scale_words(p.k_nvs, it.q0 + lane + 96, p.T, p.Hkv, it.g);
            wk = make_uint4(w0.x, w1.x, w2.x, w3.x);
            wk2 = make_uint4(w0.y, w1.y, w2.y, w3.y);
          } else {
            wk.x = pt_word(p.k_spt, it.q0 + lane, p.T, p.Hkv, it.g);
            wk.y = pt_word(p.k_spt, it.q0 + lane + 32, p.T, p.Hkv, it.g);
            wk.z = pt_word(p.k_spt, it.q0 + lane + 64, p.T, p.Hkv, it.g);
            wk.w = pt_word(p.k_spt, it.q0 + lane + 96, p.T, p.Hkv, it.g);
          }
          // the scale words were read above, so that their latency overlaps this wait
          if (unit_i > 0 && !warp_wait(q_empty, (unit_i - 1) & 1, wd, 51)) { ok = false; break; }
          if (kNv) reinterpret_cast<uint4*>(sfKpt2)[lane] = wk2;
          reinterpret_cast<uint4*>(sfKpt)[lane] = wk;
          fence_proxy_async_smem();
          if (lane == 0) {
            mbar_arrive_expect_tx(kpt_full, kKBytes);
            tma_load_3d(sKpt, &tm_kpt, kpt_full, 0, it.g, it.q0);  // the diagonal key tile starts at q0
          } else {
            mbar_arrive(kpt_full);
          }
          ++kpt_loads;
        }
      }
    }
    if (lane == 0) {
      if (kpt_loads > 0) drain_wait(kpt_full, (kpt_loads - 1) & 1, p.timeout_ns);
      for (uint32_t i = (kv_it > kSlots ? kv_it - kSlots : 0); i < kv_it; ++i)
        drain_wait(kv_full + (i % kSlots), (i / kSlots) & 1, p.timeout_ns);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t aq = smem_u32(sQ), akpt = smem_u32(sKpt), avpt = smem_u32(sVpt), ap = smem_u32(sP),
                     apd = smem_u32(sPd), aring = smem_u32(sRing), asf = smem_u32(sfQ);
      uint32_t kv_it = 0, p_cnt = 0, o_used = 0;
      int unit_i = 0;
      bool ok = true;
      auto kslot_of = [&](int j) { return (int)((kv_it + 2 * j) % kSlots); };
      auto vslot_of = [&](int j) { return (int)((kv_it + 2 * j + 1) % kSlots); };
      auto wait_slot = [&](int j, int kv) {
        const uint32_t idx = kv_it + 2 * j + kv;
        return mbar_wait(kv_full + (idx % kSlots), (idx / kSlots) & 1, wd, 53);
      };
      // S (into buffer col) = Q K^T with K codes at `kaddr` and its scales at TMEM column sfb
      // descriptors built once per operand tile and advanced by constant
      // offsets (start address >> 4 in the low field)
      const uint64_t dq = sdesc_sw128(aq, 16, 1024), dp = sdesc_sw128(ap, 16, 1024);
      // (mixed path: two NVFP4 MMAs of K = 64, scale words of channels
      // 0..63 at sfb and 64..127 at sfb2; both tiles 64-byte swizzled)
      auto issue_s = [&](uint32_t col, uint32_t kaddr, uint32_t sfb, uint32_t sfb2) {
        if constexpr (kNv) {
          const uint64_t dqn = sdesc_sw64(aq), dkn = sdesc_sw64(kaddr);
          constexpr uint32_t idn = idesc_nvf4(128, 128);
          mma_nvf4_ss(tmem + col, dqn, dkn, idn, tmem + kSfQ, tmem + sfb, 0u);
          mma_nvf4_ss(tmem + col, dqn + 2, dkn + 2, idn, tmem + kSfQ2, tmem + sfb2, 1u);  // +32 bytes
        } else {
          const uint64_t dk = sdesc_sw128(kaddr, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_mxf8_ss(tmem + col, dq + ((kk * 32) >> 4), dk + ((kk * 32) >> 4), idesc_mxf8(128, 128, false, kk, kk),
                        (tmem + kSfQ) | ((uint32_t)kk << 30), (tmem + sfb) | ((uint32_t)kk << 30), kk > 0);
        }
      };
      auto issue_s_tile = [&](int j, uint32_t col) {
        const int ks = kslot_of(j);
        const uint32_t sk = (j & 1) ? kSfK1 : kSfK, sk2 = (j & 1) ? kSfK21 : kSfK2;
        tmem_cp_sf(tmem + sk, asf + (3 + ks) * kSfBlk);
        if constexpr (kNv) tmem_cp_sf(tmem + sk2, smem_u32(sfRing2) + ks * kSfBlk);
        issue_s(col, aring + ks * kCodeTile, sk, sk2);
      };
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_take(ring, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const Item it = decode(p, un);
        const int n = it.n;
        if (!mbar_wait(q_full, unit_i & 1, wd, 54)) break;
        tc_fence_after();
        tmem_cp_sf(tmem + kSfQ, asf);
        if constexpr (kNv) tmem_cp_sf(tmem + kSfQ2, smem_u32(smem + oSf2));
        // the diagonal per-token K (and its scales) arrive on their own barrier
        auto wait_kpt = [&]() {
          if (!mbar_wait(kpt_full, unit_i & 1, wd, 61)) return false;
          tc_fence_after();
          tmem_cp_sf(tmem + kSfKpt, asf + kSfBlk);
          if constexpr (kNv) tmem_cp_sf(tmem + kSfKpt2, smem_u32(sfKpt2));
          return true;
        };
        // prologue: S(0) (+ per-token S if tile 0 is the diagonal), S(1)
        if (!wait_slot(0, 0)) break;
        tc_fence_after();
        issue_s_tile(0, kS0);
        if (n == 1) {
          if (!wait_kpt()) break;
          issue_s(kS1, akpt, kSfKpt, kSfKpt2);
        }
        tc_commit(s_full + 0);
        tc_commit(kv_empty + kslot_of(0));
        if (n >= 2) {
          if (!wait_slot(1, 0)) break;
          tc_fence_after();
          issue_s_tile(1, kS1);
          if (n > 2) tc_commit(s_full + 1);  // the diagonal tile commits after its per-token S
          tc_commit(kv_empty + kslot_of(1));
        }
        for (int j = 0; j < n; ++j) {
          if (!mbar_wait(p_full, p_cnt & 1, wd, 55)) { ok = false; break; }
          ++p_cnt;
          if (!wait_slot(j, 1)) { ok = false; break; }
          if (j == 0 && o_used > 0 && !mbar_wait(o_free, (o_used - 1) & 1, wd, 56)) { ok = false; break; }
          tc_fence_after();
          const int vs = vslot_of(j);
          tmem_cp_sf(tmem + kSfP, asf + 2 * kSfBlk);
          tmem_cp_sf(tmem + kSfV, asf + (3 + vs) * kSfBlk);
          const uint64_t dv = sdesc_sw128(aring + vs * kCodeTile, 16384, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_mxf8_ss(tmem + kO, dp + ((kk * 32) >> 4), dv + ((kk * 4096) >> 4), idesc_mxf8(128, 128, true, kk, kk),
                        (tmem + kSfP) | ((uint32_t)kk << 30), (tmem + kSfV) | ((uint32_t)kk << 30),
                        (j > 0 || kk > 0) ? 1u : 0u);
          if (j == n - 1) {
            // diagonal 32x32 blocks: exact bf16 P~ times dequantised per-token V
            if (!mbar_wait(vd_full, unit_i & 1, wd, 62)) { ok = false; break; }
            tc_fence_after();
            constexpr uint32_t idesc_d = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_f16_ss(tmem + kO, sdesc_sw128(apd + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024),
                         sdesc_sw128(avpt + kk * 2048, kBox, 1024), idesc_d, 1u);
          }
          tc_commit(pv_done);
          tc_commit(kv_empty + vs);
          if (j == n - 1) {
            tc_commit(o_full);
            ++o_used;
          }
          if (j + 2 < n) {
            if (!wait_slot(j + 2, 0)) { ok = false; break; }
            tc_fence_after();
            issue_s_tile(j + 2, (j & 1) ? kS1 : kS0);
            if (j + 2 < n - 1) tc_commit(s_full + (j & 1));
            tc_commit(kv_empty + kslot_of(j + 2));
          }
          if (j == n - 2) {
            // per-token S of the diagonal tile, into the buffer tile n-2 freed
            if (!wait_kpt()) { ok = false; break; }
            issue_s((j & 1) ? kS1 : kS0, akpt, kSfKpt, kSfKpt2);
            tc_commit(s_full + ((j + 1) & 1));  // signals tile n-1 = j+1
          }
        }
        if (!ok) break;
        kv_it += 2 * n;
        tc_commit(q_empty);
      }
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else if (warp < kComputeWarps) {
    // ------------------------------------------------------------ softmax
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    float* xmax = reinterpret_cast<float*>(smem + oXmax);
    float* lsum = reinterpret_cast<float*>(smem + oLsum);
    // the four warps that share this row quarter meet here (bounded wait)
    uint32_t x_cnt = 0;
    auto row_sync = [&]() {
      warp_arrive(xbar + quarter);
      const bool r = warp_wait(xbar + quarter, x_cnt & 1, wd, 60);
      ++x_cnt;
      return r;
    };
    uint32_t s_cnt[2] = {0, 0}, pv_cnt = 0, o_cnt = 0, tiles = 0;
    bool ok = true;
    // Q of an item is staged before the previous item's epilogue (its first
    // scores then overlap that epilogue), its diagonal V after it (the
    // previous item's last P V reads sVpt until o_full)
    uint32_t uk = 0;
    UnitInfo un = unit_take_warp(ring, uk++, wd);
    bool have = un.w >= 0 && un.w < n_units;
    if (have) {
      stage_q<kNv>(p, decode(p, un), row, wg, smem + oQ, smem + oSf);
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(q_full);
    }
    while (have && ok) {
      const Item it = decode(p, un);
      const int n = it.n;
      const int q_idx = it.q0 + row;
      stage_v(p, it, row, wg, smem + oVpt);
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(vd_full);
      UnitInfo nx{-1, 0, 0, 0, 0, 0};
      bool have_next = false;
      float M = -INFINITY, l = 0.f;  // l: this thread's share of the row sum
      for (int j = 0; j < n; ++j, ++tiles) {
        if (j == n - 1) {
          // the next item, taken now so that its Q reaches L2 during this tile
          nx = unit_take_warp(ring, uk++, wd);
          have_next = nx.w >= 0 && nx.w < n_units;
          if (have_next) prefetch_item(p, decode(p, nx), row, wg);
        }
        const int sbi = j & 1;
        if (!warp_wait(s_full + sbi, (sbi ? s_cnt[1] : s_cnt[0]) & 1, wd, 57)) { ok = false; break; }
        if (sbi) ++s_cnt[1]; else ++s_cnt[0];
        tc_fence_after();
        const bool diag = j == n - 1;
        // on the diagonal tile key block `quarter` is this row's own block
        // (per-token scores, from the other buffer); later blocks are future keys
        const bool own = diag && wg == quarter;
        const bool future = diag && wg > quarter;
        uint32_t r[32];
        if (!future) {
          tmem_ld32(lane_base + (own ? ((j & 1) ? kS0 : kS1) : ((j & 1) ? kS1 : kS0)) + 32 * wg, r);
          tmem_wait_ld(r);
        }
        // raw scores, -inf where not visible (masks only on the diagonal tile)
        float x[32];
        if (future) {
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = -INFINITY;
        } else if (own) {
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = c <= lane ? __uint_as_float(r[c]) : -INFINITY;
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(r[c]);
        }
        // block maximum of the raw scores (the scale is positive), in log2 units
        float pm[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) pm[k] = fmaxf(x[k], x[4 + k]);
#pragma unroll
        for (int c = 8; c < 32; c += 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k) pm[k] = fmax3(pm[k], x[c + k], x[c + 4 + k]);
        }
        const float bmax = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])) * p.scale_log2;
        float* xm = xmax + (tiles & 1) * 512;
        xm[wg * 128 + row] = bmax;
        if (!row_sync()) { ok = false; break; }
        const float mx = fmaxf(fmaxf(xm[row], xm[128 + row]), fmaxf(xm[256 + row], xm[384 + row]));
        float alpha = 1.f;
        if (mx > M + kRescaleThreshold) {
          const float Mn = ceilf(mx);
          // 2^(M - Mn), built exactly (0 on the first tile, when M = -inf)
          const float dk = M - Mn;
          alpha = (dk >= -126.f) ? mx_pow2((int)dk) : 0.f;
          l *= alpha;
          M = Mn;
        }
        const bool any_rescale = __any_sync(0xFFFFFFFFu, alpha != 1.f) && j > 0;
        // u = 2^(s scale log2(e) - M) with one FMA per element; row sum
        // before quantisation and block maximum of u in four partial chains
        // each; MX quantisation of the block
        // (packed pairs: one FMA per pair for the arguments, one add per pair
        // for the row sum, and the block quantisation on pairs)
        uint64_t u2[16], rs2[2] = {0ull, 0ull};
        {
          const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2), nM2 = f2_pack(-M, -M);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float a, b;
            f2_unpack(f2_fma(f2_pack(x[2 * c], x[2 * c + 1]), sl2, nM2), a, b);
            u2[c] = f2_pack(fast_exp2(a), fast_exp2(b));
            rs2[c & 1] = (c < 2) ? u2[c] : f2_add(rs2[c & 1], u2[c]);
          }
          float s0, s1, s2, s3;
          f2_unpack(rs2[0], s0, s1);
          f2_unpack(rs2[1], s2, s3);
          l += (s0 + s1) + (s2 + s3);
        }
        uint32_t codes[8];
        const int X = (int)mx_quant32_pairs<true>(u2, p.rule, codes) - 127;
        // bf16 copy of the own block's P~ (exact); its FP8 codes are zeroed
        uint32_t pd[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) pd[c] = 0;
        if (own) {
          const float scd = mx_pow2(X < -126 ? -126 : X);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float a, b, cc, d;
            mx_decode2(codes[c] & 0xFFFFu, a, b);
            mx_decode2(codes[c] >> 16, cc, d);
            pd[2 * c] = pack_bf16x2(a * scd, b * scd);
            pd[2 * c + 1] = pack_bf16x2(cc * scd, d * scd);
            codes[c] = 0;
          }
        }
        // PV(j-1) must be done before P's shared buffer and O are touched
        if (j > 0) {
          if (!warp_wait(pv_done, pv_cnt & 1, wd, 58)) { ok = false; break; }
          ++pv_cnt;
          tc_fence_after();
        }
        // P codes: row `row`, 16-byte chunks 2 wg, 2 wg + 1 (128-byte swizzle)
        {
          uint8_t* prow = sP + row * 128;
          *reinterpret_cast<uint4*>(prow + (((2 * wg) ^ (row & 7)) << 4)) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
          *reinterpret_cast<uint4*>(prow + (((2 * wg + 1) ^ (row & 7)) << 4)) = make_uint4(codes[4], codes[5], codes[6], codes[7]);
          sfP[(row & 31) * 16 + (row >> 5) * 4 + wg] = (uint8_t)(X + 127);
        }
        if (diag) {
          // P_diag: bf16, two 64-key boxes of 128 rows x 128 bytes; only the own block is non-zero
          const int box = wg >> 1, c0 = (wg & 1) * 4;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(sPd + box * kBox + row * 128 + (((c0 + c) ^ (row & 7)) << 4)) =
                make_uint4(pd[4 * c], pd[4 * c + 1], pd[4 * c + 2], pd[4 * c + 3]);
        }
        if (any_rescale) {
          uint32_t t[32];
          tmem_ld32(lane_base + kO + 32 * wg, t);
          tmem_wait_ld(t);
#pragma unroll
          for (int e = 0; e < 32; ++e) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
          tmem_st32(lane_base + kO + 32 * wg, t);
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive(p_full);
      }
      if (!ok) break;
      if (have_next) {
        // every S MMA of this item has completed (its last scores were read
        // above), so sQ and sfQ may take the next item's Q
        stage_q<kNv>(p, decode(p, nx), row, wg, smem + oQ, smem + oSf);
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive(q_full);
      }
      // epilogue: the row sum from the four block shares, O columns [32 wg, 32 wg + 32)
      lsum[wg * 128 + row] = l;
      if (!row_sync()) break;
      const float lt = (lsum[row] + lsum[128 + row]) + (lsum[256 + row] + lsum[384 + row]);
      if (!warp_wait(o_full, o_cnt & 1, wd, 59)) break;
      ++o_cnt;
      ++pv_cnt;  // the last tile's PV completion is covered by o_full
      tc_fence_after();
      const float inv_l = 1.f / lt;
      const bool valid = q_idx < it.e && 32 * wg < p.d;
      {
        uint32_t t[32];
        tmem_ld32(lane_base + kO + 32 * wg, t);
        tmem_wait_ld(t);
        uint32_t ob[16], rb[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float f0 = __uint_as_float(t[2 * e]) * inv_l, f1 = __uint_as_float(t[2 * e + 1]) * inv_l;
          ob[e] = pack_bf16x2(f0, f1);
          rb[e] = pack_bf16x2(f0 - __uint_as_float(ob[e] << 16), f1 - __uint_as_float(ob[e] & 0xFFFF0000u));
        }
        if (valid) {
          __nv_bfloat16* orow = p.o + ((size_t)q_idx * p.Hq + it.h) * p.d + 32 * wg;
          __nv_bfloat16* rrow = p.o_resid ? p.o_resid + ((size_t)q_idx * p.Hq + it.h) * p.d + 32 * wg : nullptr;
          if (p.wide) {
            st_global_32B(orow, ob);
            st_global_32B(orow + 16, ob + 8);
            if (rrow) {
              st_global_32B(rrow, rb);
              st_global_32B(rrow + 16, rb + 8);
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(ob[4 * e], ob[4 * e + 1], ob[4 * e + 2], ob[4 * e + 3]);
            if (rrow) {
              uint4* rdst = reinterpret_cast<uint4*>(rrow);
#pragma unroll
              for (int e = 0; e < 4; ++e) rdst[e] = make_uint4(rb[4 * e], rb[4 * e + 1], rb[4 * e + 2], rb[4 * e + 3]);
            }
          }
        }
      }
      tc_fence_before();
      warp_arrive(o_free);
      if (q_idx < it.e && wg == 0) p.lse[(size_t)it.h * p.T + q_idx] = (M + __log2f(lt)) * kLn2;
      un = nx;
      have = have_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) p.cta_times[2 + 2 * blockIdx.x] = globaltimer_ns();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_fwd_mxfp8(const FwdMxArgs& a, cudaStream_t stream) {
  CUtensorMap tktb, tkpt, tvtb;
  if (a.nv) {
    if (!make_tmap_nv(&tktb, a.k_nvv, a.T, a.Hkv) || !make_tmap_nv(&tkpt, a.k_nvv, a.T, a.Hkv))
      return cudaErrorInvalidValue;
  } else if (!make_tmap_codes(&tktb, a.k_vtb, a.T, a.Hkv) || !make_tmap_codes(&tkpt, a.k_vpt, a.T, a.Hkv)) {
    return cudaErrorInvalidValue;
  }
  if (!make_tmap_codes(&tvtb, a.v_vtb, a.T, a.Hkv)) return cudaErrorInvalidValue;
  const auto kern = a.nv ? fwd_mxfp8_kernel<true> : fwd_mxfp8_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  Params p;
  p.cu = a.cu;
  p.sched = sched_view(a.sched);
  p.cta_times = a.cta_times[0];
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.q_vpt = a.q_vpt;
  p.q_spt = a.q_spt;
  p.q_vtb = a.q_vtb;
  p.q_stb = a.q_stb;
  p.v_vpt = a.v_vpt;
  p.v_spt = a.v_spt;
  p.k_stb = a.k_stb;
  p.k_spt = a.k_spt;
  p.v_stb = a.v_stb;
  p.k_nvs = a.k_nvs;
  p.q_nvv = a.q_nvv;
  p.q_nvs = a.q_nvs;
  p.nv_g_q = a.nv_g_q;
  p.nv_six_g_q = 6.0f * a.nv_g_q;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.o_resid = static_cast<__nv_bfloat16*>(a.o_resid);
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.T = a.T;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.d = a.d;
  p.n_docs = a.n_docs;
  // mixed path: the scores' MMAs leave out the decode scales of Q and K
  p.scale_log2 = a.scale * 1.4426950408889634f * (a.nv ? a.nv_g_q * a.nv_g_k : 1.f);
  p.rule = a.rule;
  p.wide = aligned32(a.o) && aligned32(a.o_resid);
  const long long max_units = (long long)a.sched.max_items * a.Hq;
  const int grid = (int)(max_units < a.num_sms ? max_units : a.num_sms);
  kern<<<grid, kThreads, kSmemBytes, stream>>>(tktb, tkpt, tvtb, p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace fapk
