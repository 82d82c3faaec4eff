// Forward of causal packed-document attention, bf16 operands, for sm_100a.
//
// Computes, per query head and document, S = scale Q K^T, the causal and
// document mask, an online softmax and O = P V, with S and P kept on chip
// ("GPT Kernel Programlama: MatMul, Softmax ve Attention Hesabi" secs. 3-7;
// "FlashAttention (HU)" secs. "Tiling es blokkos feldolgozas", "Online
// Softmax-szamitas", "Muveletek osszevonasa egyetlen CUDA-kernelbe").
//
// Design (one persistent CTA per SM, 384 threads):
//  * work item = (document, pair of 128-row query tiles, head), taken from the
//    cost-ordered list of the scheduler; query tiles and key tiles are aligned
//    to the document start, so only the last key tile of a query tile needs
//    the causal mask and no tile ever spans two documents' keys for a valid
//    query row (rows past the document end are computed and discarded);
//  * warp 8 (one lane): TMA loads of Q0/Q1 once per item and of K_j into a
//    ring of shared-memory slots; warp 11 (one lane): V_j into a ring of its
//    own, so that K loads never queue behind a V slot (128-byte swizzle);
//  * warps 9 and 10 (one lane each): tcgen05 MMAs of query tile 0 and of query
//    tile 1.  S_i = Q_i K_j^T (bf16, both operands K-major in shared memory)
//    into TMEM; O_i += P_i V_j in fp16 with P_i in shared memory (K-major,
//    128-byte swizzle) and V_j MN-major (the fp16 copy of V made by the
//    prepass).  The softmax releases S_i as soon as it has read it, so
//    S_i(j+1) is computed while P_i(j) is formed, and the two issuing threads
//    keep one tile's MMAs queued while the other waits.  fp16 keeps 11
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

constexpr int kThreads = 384;
constexpr int kLoadWarp = 8;    // Q, K
constexpr int kMmaWarp = 9;     // query tile 0 (warp 10: query tile 1); owns the TMEM allocation
constexpr int kVLoadWarp = 11;  // V
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct Cfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxBytes = 128 * 64 * 2;
  static constexpr int kNumBox = D / 64;
  // K runs one tile ahead of V; P of both query tiles (128 x 128 fp16, two
  // 64-key boxes) in shared memory
  static constexpr int kKStages = (D == 128) ? 2 : 3, kVStages = (D == 128) ? 1 : 2;
  static constexpr int kPBytes = 128 * 128 * 2;
  static constexpr int kSmemTiles = (2 + kKStages + kVStages) * kTileBytes + 2 * kPBytes;
  static constexpr uint32_t kSCol0 = 0, kSCol1 = 128;
  static constexpr uint32_t kOCol0 = 256, kOCol1 = 256 + D;
  static constexpr uint32_t kTmemCols = 512;
  // barriers: q_full, q_empty, k_full[K], k_empty[K], v_full[V], v_empty[V],
  // s_full[2], s_free[2], p_full[2], p_free[2], o_full[2], o_free[2], fin
  // + the unit ring's full[8] and empty[8]
  static constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVStages + 12 + 1 + 2 * kUnitRing;
  static constexpr int kSmemBytes = kSmemTiles + kNumBars * 8 + 16 + kUnitRingBytes + 1024;
};
static_assert(Cfg<128>::kSmemBytes <= 227 * 1024 && Cfg<64>::kSmemBytes <= 227 * 1024,
              "shared memory of the forward exceeds the 227 KB a CTA may use");

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
  int wide;  // O and its residual 32-byte aligned: 32-byte stores
  unsigned long long* cta_times;  // per-CTA (start, end) records, or null
};

struct Item {
  int s, e, u, h, g, q0, n0, n1, nkv;
};

__device__ __forceinline__ Item decode(const Params& p, const UnitInfo& un) {
  Item it;
  it.u = un.tile;
  it.h = un.h;
  it.g = it.h / (p.Hq / p.Hkv);
  it.s = un.s;
  it.e = un.e;
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                 // 2 tiles
  uint8_t* sK = smem + 2 * C::kTileBytes;             // K ring
  uint8_t* sV = sK + C::kKStages * C::kTileBytes;     // V ring
  uint8_t* sP = sV + C::kVStages * C::kTileBytes;     // P_0, P_1
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemTiles);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + C::kKStages;
  uint64_t* v_full = k_empty + C::kKStages;
  uint64_t* v_empty = v_full + C::kVStages;
  uint64_t* s_full = v_empty + C::kVStages;  // [2] each
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_full + 4;
  uint64_t* p_free = s_full + 6;
  uint64_t* o_full = s_full + 8;
  uint64_t* o_free = s_full + 10;
  uint64_t* fin = s_full + 12;
  const UnitRing ring{reinterpret_cast<int*>(bars + C::kNumBars) + 4, bars + C::kNumBars - 2 * kUnitRing,
                      bars + C::kNumBars - kUnitRing};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);  // both MMA threads
    for (int i = 0; i < C::kKStages; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 2);
    }
    for (int i = 0; i < C::kVStages; ++i) {
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 2);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, 4);  // the tile's four softmax warps
      mbar_init(p_full + i, 4);
      mbar_init(p_free + i, 1);
      mbar_init(o_full + i, 1);
      mbar_init(o_free + i, 128);
    }
    mbar_init(fin, 2);
    unit_ring_init(ring, 3 + 8);  // the V loader, both MMA threads and the 8 softmax warps
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
    // ------------------------------------------------------------ TMA loads: Q, K
    if (lane == 0) {
      uint32_t kt = 0;
      int unit_i = 0;
      int last_q_phase = -1;
      bool ok = true;
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_produce(ring, us, p.cu, p.sched.next, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const Item it = decode(p, un);
        if (unit_i > 0 && !mbar_wait(q_empty, (unit_i - 1) & 1, wd, 1)) break;
        mbar_arrive_expect_tx(q_full, (it.n1 ? 2 : 1) * C::kTileBytes);
        last_q_phase = unit_i & 1;
        for (int b = 0; b < C::kNumBox; ++b) {
          tma_load_3d(sQ + b * C::kBoxBytes, &tm_q, q_full, 64 * b, it.h, it.q0);
          if (it.n1) tma_load_3d(sQ + C::kTileBytes + b * C::kBoxBytes, &tm_q, q_full, 64 * b, it.h, it.q0 + 128);
        }
        for (int j = 0; j < it.nkv; ++j, ++kt) {
          const int slot = kt % C::kKStages;
          const uint32_t use = kt / C::kKStages;
          if (use > 0 && !mbar_wait(k_empty + slot, (use - 1) & 1, wd, 2)) { ok = false; break; }
          mbar_arrive_expect_tx(k_full + slot, C::kTileBytes);
          for (int b = 0; b < C::kNumBox; ++b)
            tma_load_3d(sK + slot * C::kTileBytes + b * C::kBoxBytes, &tm_k, k_full + slot, 64 * b, it.g,
                        it.s + 128 * j);
        }
      }
      // teardown: let the copies this thread issued land before the CTA exits
      const uint64_t budget = p.timeout_ns;
      if (last_q_phase >= 0) drain_wait(q_full, (uint32_t)last_q_phase, budget);
      for (uint32_t i = (kt > C::kKStages ? kt - C::kKStages : 0); i < kt; ++i)
        drain_wait(k_full + (i % C::kKStages), (i / C::kKStages) & 1, budget);
    }
  } else if (warp == kVLoadWarp) {
    // ------------------------------------------------------------ TMA loads: V
    if (lane == 0) {
      uint32_t vt = 0;
      bool ok = true;
      for (uint32_t uk = 0; ok; ++uk) {
        const UnitInfo un = unit_take(ring, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const Item it = decode(p, un);
        for (int j = 0; j < it.nkv; ++j, ++vt) {
          const int slot = vt % C::kVStages;
          const uint32_t use = vt / C::kVStages;
          if (use > 0 && !mbar_wait(v_empty + slot, (use - 1) & 1, wd, 11)) { ok = false; break; }
          mbar_arrive_expect_tx(v_full + slot, C::kTileBytes);
          // injected fault: the CTA that takes the first (longest) unit drops its second V copy
          const bool drop = (p.flags & FAPK_FLAG_INJECT_DROP_LOAD) && w == 0 && j == 1;
          if (!drop) {
            for (int b = 0; b < C::kNumBox; ++b)
              tma_load_3d(sV + slot * C::kTileBytes + b * C::kBoxBytes, &tm_v, v_full + slot, 64 * b, it.g,
                          it.s + 128 * j);
          }
        }
      }
      for (uint32_t i = (vt > C::kVStages ? vt - C::kVStages : 0); i < vt; ++i)
        drain_wait(v_full + (i % C::kVStages), (i / C::kVStages) & 1, p.timeout_ns);
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // ------------------------------------------------------------ MMA issue, query tile i
    // Both threads walk every K and V slot use of an item in the loaders'
    // order; a thread releases a use after its fill completed, also when it
    // does not read it, so that no release lands a phase early.
    if (lane == 0) {
      const int i = warp - kMmaWarp;
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, D, false, true);
      const uint32_t sk_addr = smem_u32(sK), sv_addr = smem_u32(sV);
      // descriptors: base + (byte offset >> 4) in the start-address field; a
      // step of K = 16 is 32 bytes inside a 128-byte swizzle row, 16 KB across
      // 64-element boxes
      const uint64_t dq = sdesc_sw128(smem_u32(sQ) + i * C::kTileBytes, 16, 1024);
      const uint64_t dp = sdesc_sw128(smem_u32(sP) + i * C::kPBytes, 16, 1024);
      const uint32_t scol = tmem + (i ? C::kSCol1 : C::kSCol0), ocol = tmem + (i ? C::kOCol1 : C::kOCol0);
      uint32_t kt = 0, vt = 0, s_uses = 0, pv = 0, o_used = 0;
      int unit_i = 0;
      bool ok = true;
      // next K slot: S_i = Q_i K^T into TMEM once the softmax has read S_i out
      auto step_k = [&](bool use) {
        const int slot = kt % C::kKStages;
        if (!mbar_wait(k_full + slot, (kt / C::kKStages) & 1, wd, 4)) return false;
        if (use) {
          if (s_uses > 0 && !mbar_wait(s_free + i, (s_uses - 1) & 1, wd, 12)) return false;
          tc_fence_after();
          const uint64_t db = sdesc_sw128(sk_addr + slot * C::kTileBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
            mma_f16_ss(scol, dq + off, db + off, idesc_qk, kk > 0);
          }
          tc_commit(s_full + i);
          ++s_uses;
        }
        tc_commit(k_empty + slot);
        ++kt;
        return true;
      };
      // next V slot: O_i += P_i V (8 MMAs of K = 16 keys; V MN-major, 16 keys =
      // 2048 bytes per step, 64-channel chunks 16 KB apart)
      auto step_v = [&](bool use, bool acc, bool first, bool last) {
        const int slot = vt % C::kVStages;
        if (!mbar_wait(v_full + slot, (vt / C::kVStages) & 1, wd, 5)) return false;
        if (use) {
          if (first && o_used > 0 && !mbar_wait(o_free + i, (o_used - 1) & 1, wd, 6)) return false;
          if (!mbar_wait(p_full + i, pv & 1, wd, 7)) return false;
          tc_fence_after();
          const uint64_t dv = sdesc_sw128(sv_addr + slot * C::kTileBytes, C::kBoxBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
            mma_f16_ss(ocol, dp + off, dv + ((kk * 2048) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
          }
          tc_commit(p_free + i);  // P_i's buffer may be rewritten, O_i is settled
          ++pv;
          if (last) {
            tc_commit(o_full + i);
            ++o_used;
          }
        }
        tc_commit(v_empty + slot);
        ++vt;
        return true;
      };
      for (uint32_t uk = 0; ok; ++uk, ++unit_i) {
        const UnitInfo un = unit_take(ring, uk, wd);
        const int w = un.w;
        if (w < 0 || w >= n_units) break;
        const Item it = decode(p, un);
        const int n = i ? it.n1 : it.n0;
        if (!mbar_wait(q_full, unit_i & 1, wd, 3)) break;
        if (!step_k(n > 0)) break;
        // Q is free once the item's last scores complete: the loader fetches
        // the next item's Q while this item's P V MMAs run
        if (it.nkv == 1) tc_commit(q_empty);
        for (int j = 0; j < it.nkv; ++j) {
          // the next scores go ahead of this key tile's P V
          if (j + 1 < it.nkv) {
            if (!step_k(j + 1 < n)) { ok = false; break; }
            if (j + 2 == it.nkv) tc_commit(q_empty);
          }
          if (!step_v(j < n, j > 0, j == 0, j == n - 1)) { ok = false; break; }
        }
        if (!ok) break;
      }
      // teardown: every MMA issued by this thread completes before TMEM is freed
      tc_commit(fin);
      drain_wait(fin, 0, p.timeout_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_addr = lane_base + (wg ? C::kSCol1 : C::kSCol0);
    const uint32_t o_addr = lane_base + (wg ? C::kOCol1 : C::kOCol0);
    uint8_t* prow = sP + wg * C::kPBytes + row * 128;  // this row of P_wg in box 0
    const int sw = row & 7;                            // 128-byte swizzle of the row
    uint32_t s_cnt = 0, p_cnt = 0, o_cnt = 0;
    for (uint32_t uk = 0;; ++uk) {
      const UnitInfo un = unit_take_warp(ring, uk, wd);
      const int w = un.w;
      if (w < 0 || w >= n_units) break;
      const Item it = decode(p, un);
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
        tc_fence_before();
        warp_arrive(s_free + wg);  // the next scores may overwrite S
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
        // independent partial maxima of three-operand max instructions; column
        // 0 of the last key tile is the query's own key, so the maximum is finite
        float pm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = fmaxf(x[k], x[8 + k]);
#pragma unroll
        for (int c = 16; c < 128; c += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) pm[k] = fmax3(pm[k], x[c + k], x[c + 8 + k]);
        }
        const float mx = fmaxf(fmax3(pm[0], pm[1], pm[2]), fmax3(fmax3(pm[3], pm[4], pm[5]), pm[6], pm[7])) *
                         p.scale_log2;
        const float m_new = fmaxf(m, mx);
        const bool need = m_new > m + kRescaleThreshold;
        float alpha = 1.f;
        const bool any_need = __any_sync(0xFFFFFFFFu, need);
        if (need) {
          alpha = fast_exp2(m - m_new);
          m = m_new;
          l *= alpha;
        }
        // P = 2^(s scale log2(e) - m): one packed FMA per pair of elements;
        // row sum in four independent packed partial sums
        uint32_t pk[64];
        uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
        const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-m, -m);
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          float a, b;
          f2_unpack(f2_fma(f2_pack(x[2 * c], x[2 * c + 1]), sl2, nm2), a, b);
          a = fast_exp2(a);
          b = fast_exp2(b);
          const uint64_t ab = f2_pack(a, b);
          rs2[c & 3] = (c < 4) ? ab : f2_add(rs2[c & 3], ab);
          pk[c] = pack_f16x2(a, b);
        }
        {
          float s0, s1, s2, s3;
          f2_unpack(f2_add(rs2[0], rs2[1]), s0, s1);
          f2_unpack(f2_add(rs2[2], rs2[3]), s2, s3);
          l += (s0 + s2) + (s1 + s3);
        }
        // the previous P V of this tile has completed: P's buffer is free and
        // O is settled for the rescale
        if (p_cnt > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(p_free + wg, (p_cnt - 1) & 1, wd, 13))) {
          ok = false;
          break;
        }
        ++p_cnt;
        tc_fence_after();
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
          tmem_wait_st();
        }
        // P row -> shared memory: 16-byte chunk q holds keys 8q..8q+7, chunks
        // 0-7 in box 0 and 8-15 in box 1, each placed at (q mod 8) xor (row mod 8)
#pragma unroll
        for (int q = 0; q < 16; ++q)
          *reinterpret_cast<uint4*>(prow + (q >> 3) * C::kBoxBytes + (((q & 7) ^ sw) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive(p_full + wg);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16, LSE = (m + log2 l) ln 2
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(o_full + wg, o_cnt & 1, wd, 10))) break;
      ++o_cnt;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool valid = q_idx < it.e;
      __nv_bfloat16* orow = p.o + ((size_t)q_idx * p.Hq + it.h) * D;
      // the row of O in one batch of TMEM loads and one wait
      uint32_t ot[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(o_addr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&ot[32 * c]));
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&ot[32 * c]));
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        const uint32_t* t = ot + 32 * c;
        uint32_t ob[16], rb[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float f0 = __uint_as_float(t[2 * e]) * inv_l, f1 = __uint_as_float(t[2 * e + 1]) * inv_l;
          ob[e] = pack_bf16x2(f0, f1);
          // residual: what bf16 rounding dropped (exactly representable up to bf16 rounding again)
          rb[e] = pack_bf16x2(f0 - __uint_as_float(ob[e] << 16), f1 - __uint_as_float(ob[e] & 0xFFFF0000u));
        }
        if (valid) {
          __nv_bfloat16* rrow = p.o_resid ? p.o_resid + ((size_t)q_idx * p.Hq + it.h) * D : nullptr;
          if (p.wide) {
            st_global_32B(orow + 32 * c, ob);
            st_global_32B(orow + 32 * c + 16, ob + 8);
            if (rrow) {
              st_global_32B(rrow + 32 * c, rb);
              st_global_32B(rrow + 32 * c + 16, rb + 8);
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(ob[4 * e], ob[4 * e + 1], ob[4 * e + 2], ob[4 * e + 3]);
            if (rrow) {
              uint4* rdst = reinterpret_cast<uint4*>(rrow + 32 * c);
#pragma unroll
              for (int e = 0; e < 4; ++e) rdst[e] = make_uint4(rb[4 * e], rb[4 * e + 1], rb[4 * e + 2], rb[4 * e + 3]);
            }
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
  p.wide = aligned32(a.o) && aligned32(a.o_resid);
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
