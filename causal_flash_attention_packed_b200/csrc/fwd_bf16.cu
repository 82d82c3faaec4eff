// Forward of causal packed-document attention, bf16 operands, for sm_100a.
//
// Computes, per query head and document, S = scale Q K^T, the causal and
// document mask, an online softmax and O = P V, with S and P kept on chip
// ("GPT Kernel Programlama: MatMul, Softmax ve Attention Hesabi" secs. 3-7;
// "FlashAttention (HU)" secs. "Tiling es blokkos feldolgozas", "Online
// Softmax-szamitas", "Muveletek osszevonasa egyetlen CUDA-kernelbe").
//
// Design (one persistent CTA per SM, 320 threads):
//  * work item = (document, pair of 128-row query tiles, head), taken from the
//    cost-ordered list of the scheduler; query tiles and key tiles are aligned
//    to the document start, so only the last key tile of a query tile needs
//    the causal mask and no tile ever spans two documents' keys for a valid
//    query row (rows past the document end are computed and discarded);
//  * warp 8 (one lane): TMA loads of Q0/Q1 once per item and of K_j, V_j
//    into a ring of shared-memory slots (128-byte swizzle);
//  * warp 9 (one lane): tcgen05 MMAs.  S_i = Q_i K_j^T (bf16, both operands
//    K-major in shared memory) into TMEM; O_i += P_i V_j in fp16 with P_i read
//    from TMEM (it overwrites S_i in place as packed fp16) and V_j MN-major in
//    shared memory (the fp16 copy of V made by the prepass).  fp16 keeps 11
//    significant bits of P where bf16 keeps 8; the backward's D = dO . O
//    inherits this accuracy;
//  * warps 0-3 / 4-7: softmax of query tile 0 / 1, one thread per query row
//    (one TMEM lane).  The running maximum is kept in log2 units and only
//    moved when it grows by more than 8 (P <= 2^8 in between), so the O
//    rescale in TMEM is rare; the result is exact up to rounding because the
//    final O / l uses the same reference.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [256+D,256+2D).
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "sched.cuh"

namespace fapk {

namespace {

constexpr int kThreads = 320;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct Cfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxBytes = 128 * 64 * 2;
  static constexpr int kNumBox = D / 64;
  static constexpr int kSlots = (D == 128) ? 4 : 8;
  static constexpr int kSmemTiles = (2 + kSlots) * kTileBytes;
  static constexpr uint32_t kSCol0 = 0, kSCol1 = 128;
  static constexpr uint32_t kOCol0 = 256, kOCol1 = 256 + D;
  static constexpr uint32_t kTmemCols = 512;
  // barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full[2],
  // o_full[2], o_free[2], final
  // + the unit ring's full[8] and empty[8]
  static constexpr int kNumBars = 2 + 2 * kSlots + 8 + 1 + 2 * kUnitRing;
  static constexpr int kSmemBytes = kSmemTiles + kNumBars * 8 + 16 + 4 * kUnitRing + 1024;
};

struct Params {
  const int32_t* cu;
  SchedView sched;
  __nv_bfloat16* o;
  float* lse;
  __nv_bfloat16* o_resid;
  DeviceStatus* status;
  uint64_t timeout_ns;
  int T, Hq, Hkv;
  float scale_log2;
  int flags;
  unsigned long long* cta_times;  // per-CTA (start, end) records, or null
};

struct Item {
  int s, e, u, h, g, q0, n0, n1, nkv;
};

__device__ __forceinline__ Item decode(const Params& p, const UnitSpace& us, int w) {
  Item it;
  int doc;
  unit_decode(us, w, doc, it.u, it.h);
  it.g = it.h / (p.Hq / p.Hkv);
  it.s = p.cu[doc];
  it.e = p.cu[doc + 1];
  it.q0 = it.s + 256 * it.u;
  it.n0 = 2 * it.u + 1;                               // key tiles 0..2u for query tile 0
  it.n1 = (it.q0 + 128 < it.e) ? 2 * it.u + 2 : 0;    // key tiles 0..2u+1 for query tile 1
  it.nkv = it.n1 ? it.n1 : it.n0;
  return it;
}

// 128 TMEM columns of this thread's lane -> registers, then one wait tied to
// all of them.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  tmem_ld32(taddr + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  tmem_ld32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
  tmem_ld32(taddr + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
  tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&r[64]));
  tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&r[96]));
}

// Bounded wait that ignores the abort flag (teardown: drain what is in flight).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t budget_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > budget_ns) return;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                              // 2 tiles
  uint8_t* sKV = smem + 2 * C::kTileBytes;         // kSlots tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemTiles);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = bars + 2 + C::kSlots;
  uint64_t* s_full = bars + 2 + 2 * C::kSlots;     // [2]
  uint64_t* p_full = s_full + 2;                   // [2]
  uint64_t* o_full = s_full + 4;                   // [2]
  uint64_t* o_free = s_full + 6;                   // [2]
  uint64_t* fin = s_full + 8;
  const UnitRing ring{reinterpret_cast<int*>(bars + C::kNumBars) + 4, bars + C::kNumBars - 2 * kUnitRing,
                      bars + C::kNumBars - kUnitRing};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 128);
      mbar_init(o_full + i, 1);
      mbar_init(o_free + i, 128);
    }
    mbar_init(fin, 1);
    unit_ring_init(ring, 1 + 8);  // the MMA thread and the 8 softmax warps
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
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
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      uint32_t kv_it = 0;
      int unit_i = 0;
      int last_q_phase = -1;
      for (uint32_t uk = 0;; ++uk, ++unit_i) {
        const int w = unit_produce(ring, p.sched.next, uk, wd);
        if (w < 0 || w >= n_units) break;
        const Item it = decode(p, us, w);
        if (unit_i > 0 && !mbar_wait(q_empty, (unit_i - 1) & 1, wd, 1)) break;
        mbar_arrive_expect_tx(q_full, (it.n1 ? 2 : 1) * C::kTileBytes);
        last_q_phase = unit_i & 1;
        for (int b = 0; b < C::kNumBox; ++b) {
          tma_load_3d(sQ + b * C::kBoxBytes, &tm_q, q_full, 64 * b, it.h, it.q0);
          if (it.n1) tma_load_3d(sQ + C::kTileBytes + b * C::kBoxBytes, &tm_q, q_full, 64 * b, it.h, it.q0 + 128);
        }
        bool ok = true;
        for (int j = 0; j < it.nkv && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv, ++kv_it) {
            const int slot = kv_it % C::kSlots;
            const uint32_t use = kv_it / C::kSlots;
            if (use > 0 && !mbar_wait(kv_empty + slot, (use - 1) & 1, wd, 2)) { ok = false; break; }
            mbar_arrive_expect_tx(kv_full + slot, C::kTileBytes);
            // injected fault: the CTA that takes the first (longest) unit drops its fourth copy
            const bool drop = (p.flags & FAPK_FLAG_INJECT_DROP_LOAD) && w == 0 && kv_it == 3;
            if (!drop) {
              const CUtensorMap* tm = kv ? &tm_v : &tm_k;
              for (int b = 0; b < C::kNumBox; ++b)
                tma_load_3d(sKV + slot * C::kTileBytes + b * C::kBoxBytes, tm, kv_full + slot, 64 * b, it.g,
                            it.s + 128 * j);
            }
          }
        }
        if (!ok) break;
      }
      // teardown: let the copies this thread issued land before the CTA exits
      const uint64_t budget = p.timeout_ns;
      if (last_q_phase >= 0) drain_wait(q_full, (uint32_t)last_q_phase, budget);
      for (uint32_t i = (kv_it > C::kSlots ? kv_it - C::kSlots : 0); i < kv_it; ++i)
        drain_wait(kv_full + (i % C::kSlots), (i / C::kSlots) & 1, budget);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, D, false, true);
      const uint32_t sq_addr = smem_u32(sQ), skv_addr = smem_u32(sKV);
      uint32_t kv_it = 0, p_cnt[2] = {0, 0}, o_used[2] = {0, 0};
      int unit_i = 0;
      // Descriptors are built once per tile and advanced by constant offsets
      // (start address >> 4 in the low field).
      // S_i = Q_i K^T: D/16 MMAs of K = 16 channels, 32 bytes apart inside a
      // 128-byte swizzle row, 16 KB apart across 64-channel boxes.
      const uint64_t dq0 = sdesc_sw128(sq_addr, 16, 1024), dq1 = sdesc_sw128(sq_addr + C::kTileBytes, 16, 1024);
      auto issue_s = [&](int i, int kslot) {
        const uint64_t da = i ? dq1 : dq0, db = sdesc_sw128(skv_addr + kslot * C::kTileBytes, 16, 1024);
        const uint32_t dcol = tmem + (i ? C::kSCol1 : C::kSCol0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
          mma_f16_ss(dcol, da + off, db + off, idesc_qk, kk > 0);
        }
      };
      // O_i += P_i V: 8 MMAs of K = 16 keys; P_i from TMEM (8 packed columns
      // per step), V MN-major (16 keys = 2048 bytes per step, 64-channel
      // chunks 16 KB apart).
      auto issue_pv = [&](int i, int vslot, bool acc) {
        const uint64_t dv = sdesc_sw128(skv_addr + vslot * C::kTileBytes, C::kBoxBytes, 1024);
        const uint32_t pcol = tmem + (i ? C::kSCol1 : C::kSCol0), dcol = tmem + (i ? C::kOCol1 : C::kOCol0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts(dcol, pcol + kk * 8, dv + ((kk * 2048) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
      };
      for (uint32_t uk = 0;; ++uk, ++unit_i) {
        const int w = unit_take(ring, uk, wd);
        if (w < 0 || w >= n_units) break;
        const Item it = decode(p, us, w);
        if (!mbar_wait(q_full, unit_i & 1, wd, 3)) break;
        int kslot = kv_it % C::kSlots;
        if (!mbar_wait(kv_full + kslot, (kv_it / C::kSlots) & 1, wd, 4)) break;
        tc_fence_after();
        issue_s(0, kslot);
        tc_commit(s_full + 0);
        if (it.n1) {
          issue_s(1, kslot);
          tc_commit(s_full + 1);
        }
        bool ok = true;
        for (int j = 0; j < it.nkv; ++j) {
          const int vslot = (kv_it + 1) % C::kSlots;
          if (!mbar_wait(kv_full + vslot, ((kv_it + 1) / C::kSlots) & 1, wd, 5)) { ok = false; break; }
          tc_commit(kv_empty + kslot);  // K_j free once S_0(j), S_1(j) complete
          const bool has_next = j + 1 < it.nkv;
          const int nslot = (kv_it + 2) % C::kSlots;
          bool next_ready = false;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int n = i ? it.n1 : it.n0;
            if (j < n) {
              if (j == 0 && o_used[i] > 0 && !mbar_wait(o_free + i, (o_used[i] - 1) & 1, wd, 6)) { ok = false; break; }
              if (!mbar_wait(p_full + i, p_cnt[i] & 1, wd, 7)) { ok = false; break; }
              ++p_cnt[i];
              tc_fence_after();
              issue_pv(i, vslot, j > 0);
              if (j == n - 1) {
                tc_commit(o_full + i);
                ++o_used[i];
              }
            }
            if (has_next && j + 1 < n) {
              if (!next_ready) {
                if (!mbar_wait(kv_full + nslot, ((kv_it + 2) / C::kSlots) & 1, wd, 8)) { ok = false; break; }
                tc_fence_after();
                next_ready = true;
              }
              issue_s(i, nslot);
              tc_commit(s_full + i);
            }
          }
          if (!ok) break;
          tc_commit(kv_empty + vslot);  // V_j free once PV_0(j), PV_1(j) complete
          kv_it += 2;
          kslot = nslot;
        }
        if (!ok) break;
        tc_commit(q_empty);
      }
      // teardown: every MMA issued by this thread completes before TMEM is freed
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_addr = lane_base + (wg ? C::kSCol1 : C::kSCol0);
    const uint32_t o_addr = lane_base + (wg ? C::kOCol1 : C::kOCol0);
    uint32_t s_cnt = 0, o_cnt = 0;
    for (uint32_t uk = 0;; ++uk) {
      const int w = unit_take_warp(ring, uk, wd);
      if (w < 0 || w >= n_units) break;
      const Item it = decode(p, us, w);
      const int n = wg ? it.n1 : it.n0;
      if (n == 0) continue;
      const int q_idx = it.q0 + 128 * wg + row;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(s_full + wg, s_cnt & 1, wd, 9))) { ok = false; break; }
        ++s_cnt;
        tc_fence_after();
        uint32_t r[128];
        tmem_ld128(s_addr, r);
        float x[128];
        const int key0 = it.s + 128 * j;
        if (j == n - 1) {
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = (key0 + c <= q_idx) ? __uint_as_float(r[c]) : -INFINITY;
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(r[c]);
        }
        // row maximum of the raw scores (the scale is positive) through eight
        // independent partial maxima, so that no 128-long dependency chain
        // sits between the scores' arrival and P; column 0 of the last key
        // tile is the query's own key, so the maximum is finite
        float pm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = x[k];
#pragma unroll
        for (int c = 8; c < 128; ++c) pm[c & 7] = fmaxf(pm[c & 7], x[c]);
        const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                               fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7]))) * p.scale_log2;
        const float m_new = fmaxf(m, mx);
        const bool need = m_new > m + kRescaleThreshold;
        float alpha = 1.f;
        const bool any_need = __any_sync(0xFFFFFFFFu, need);
        if (need) {
          alpha = fast_exp2(m - m_new);
          m = m_new;
          l *= alpha;
        }
        // P = 2^(s scale log2(e) - m) with one FMA per element; row sum in
        // four independent partial sums
        uint32_t pk[64];
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
        const float nm = -m;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float a = fast_exp2(fmaf(x[2 * c], p.scale_log2, nm));
          const float b = fast_exp2(fmaf(x[2 * c + 1], p.scale_log2, nm));
          rs[c & 3] += a + b;
          pk[c] = pack_f16x2(a, b);
        }
        l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
        tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        if (any_need && j > 0) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t t[32];
            tmem_ld32(o_addr + 32 * c, t);
            tmem_wait_ld(t);
#pragma unroll
            for (int e = 0; e < 32; ++e) t[e] = __float_as_uint(__uint_as_float(t[e]) * alpha);
            tmem_st32(o_addr + 32 * c, t);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + wg);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16, LSE = (m + log2 l) ln 2
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(o_full + wg, o_cnt & 1, wd, 10))) break;
      ++o_cnt;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool valid = q_idx < it.e;
      __nv_bfloat16* orow = p.o + ((size_t)q_idx * p.Hq + it.h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t t[32];
        tmem_ld32(o_addr + 32 * c, t);
        tmem_wait_ld(t);
        uint32_t ob[16], rb[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float f0 = __uint_as_float(t[2 * e]) * inv_l, f1 = __uint_as_float(t[2 * e + 1]) * inv_l;
          ob[e] = pack_bf16x2(f0, f1);
          // residual: what bf16 rounding dropped (exactly representable up to bf16 rounding again)
          rb[e] = pack_bf16x2(f0 - __uint_as_float(ob[e] << 16), f1 - __uint_as_float(ob[e] & 0xFFFF0000u));
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(ob[4 * e], ob[4 * e + 1], ob[4 * e + 2], ob[4 * e + 3]);
          if (p.o_resid) {
            uint4* rdst = reinterpret_cast<uint4*>(p.o_resid + ((size_t)q_idx * p.Hq + it.h) * D + 32 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e) rdst[e] = make_uint4(rb[4 * e], rb[4 * e + 1], rb[4 * e + 2], rb[4 * e + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(o_free + wg);
      if (valid) p.lse[(size_t)it.h * p.T + q_idx] = (m + __log2f(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.cta_times && threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) p.cta_times[2 + 2 * blockIdx.x] = globaltimer_ns();
  if (warp == kMmaWarp) tmem_dealloc(tmem, C::kTmemCols);
}

template <int D>
cudaError_t launch_d(const FwdArgs& a, cudaStream_t stream) {
  using C = Cfg<D>;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_thd(&tq, a.q, a.T, a.Hq, D) || !make_tmap_thd(&tk, a.k, a.T, a.Hkv, D) ||
      !make_tmap_thd(&tv, a.v16, a.T, a.Hkv, D, true))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  Params p;
  p.cu = a.cu;
  p.sched = sched_view(a.sched);
  p.cta_times = a.cta_times[0];
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.o_resid = static_cast<__nv_bfloat16*>(a.o_resid);
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.T = a.T;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.flags = a.flags;
  const long long max_units = (long long)a.sched.max_items * a.Hq;
  const int grid = (int)(max_units < a.num_sms ? max_units : a.num_sms);
  fwd_bf16_kernel<D><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(const FwdArgs& a, cudaStream_t stream) {
  return a.d == 128 ? launch_d<128>(a, stream) : launch_d<64>(a, stream);
}

}  // namespace fapk
