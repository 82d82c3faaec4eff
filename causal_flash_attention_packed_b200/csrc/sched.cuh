// Device side of the work order (schedule.cu): unit numbering and the
// per-CTA ring through which one loader thread hands the units it takes from
// the global counter to the CTA's other roles.
#pragma once

#include "internal.h"
#include "ptx.cuh"

namespace fapk {

// Work units of one order: documents x heads x tiles.
struct UnitSpace {
  SchedView s;
  int n_docs;   // documents with at least one tile
  int n_tiles;  // tiles in all
  int H;        // heads per unit kind (query heads, or KV heads for key tiles)
  int mode;     // kSchedQ or kSchedKV
  __device__ int n_units() const { return n_tiles * H; }
};

__device__ __forceinline__ UnitSpace unit_space(const SchedView& s, int H, int mode) {
  UnitSpace u;
  u.s = s;
  u.n_docs = s.counts[0];
  u.n_tiles = s.counts[1];
  u.H = H;
  u.mode = mode;
  return u;
}

// Unit w -> (document, tile, head).  The units of sorted document i start at
// its first tile index times H; inside, head-major, each head's tiles in
// decreasing order of work.
__device__ __forceinline__ void unit_decode(const UnitSpace& u, int w, int& doc, int& tile, int& h) {
  int lo = 0, hi = u.n_docs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (u.s.docs[mid].y * u.H <= w) lo = mid; else hi = mid - 1;
  }
  const int2 d = u.s.docs[lo];
  const int t_end = (lo + 1 < u.n_docs) ? u.s.docs[lo + 1].y : u.n_tiles;
  const int nt = t_end - d.y;
  const int local = w - d.y * u.H;
  h = local / nt;
  const int r = local - h * nt;
  doc = d.x;
  tile = (u.mode == kSchedQ) ? nt - 1 - r : r;
}

// A unit as the roles use it: its index, (document, tile, head) and the
// document's token range [s, e).
struct UnitInfo {
  int w, doc, tile, h, s, e;
};

// Ring of decoded units in shared memory: one producer thread takes the next
// unit from the global counter, decodes it once (a binary search over the
// document table and two cu_seqlens loads, all global-memory latency) and
// every other role reads the decoded entry, so that no role repeats that
// chain of dependent loads at a unit boundary.  Each role consumes each entry
// once; the entry past the last unit (index >= n_units) ends every role.
constexpr int kUnitRing = 8;
constexpr int kUnitSlotInts = 8;                              // one UnitInfo, padded to 32 bytes
constexpr int kUnitRingBytes = 4 * kUnitSlotInts * kUnitRing;  // shared-memory bytes of the entries

struct UnitRing {
  int* ids;         // [kUnitRing][kUnitSlotInts]
  uint64_t* full;   // [kUnitRing], 1 arrival (the producer)
  uint64_t* empty;  // [kUnitRing], one arrival per consumer (thread or warp)
};

__device__ __forceinline__ void unit_ring_init(const UnitRing& r, int consumers) {
  for (int i = 0; i < kUnitRing; ++i) {
    mbar_init(r.full + i, 1);
    mbar_init(r.empty + i, consumers);
  }
}

__device__ __forceinline__ UnitInfo unit_read(const UnitRing& r, int slot) {
  const volatile int* e = r.ids + kUnitSlotInts * slot;
  return UnitInfo{e[0], e[1], e[2], e[3], e[4], e[5]};
}

// Producer (one thread): the k-th unit of this CTA, decoded.  w = -1 if a
// wait gave up.
__device__ __forceinline__ UnitInfo unit_produce(const UnitRing& r, const UnitSpace& us, const int32_t* cu,
                                                 int* next, uint32_t k, const Watchdog& wd) {
  UnitInfo u{-1, 0, 0, 0, 0, 0};
  const int slot = k % kUnitRing;
  const uint32_t use = k / kUnitRing;
  if (use > 0 && !mbar_wait(r.empty + slot, (use - 1) & 1, wd, 90)) return u;
  u.w = atomicAdd(next, 1);
  if (u.w >= 0 && u.w < us.n_units()) {
    unit_decode(us, u.w, u.doc, u.tile, u.h);
    u.s = cu[u.doc];
    u.e = cu[u.doc + 1];
  }
  int* e = r.ids + kUnitSlotInts * slot;
  e[0] = u.w;
  e[1] = u.doc;
  e[2] = u.tile;
  e[3] = u.h;
  e[4] = u.s;
  e[5] = u.e;
  mbar_arrive(r.full + slot);
  return u;
}

// Producer, a whole warp: lane 0 produces, every lane returns the entry.
__device__ __forceinline__ UnitInfo unit_produce_warp(const UnitRing& r, const UnitSpace& us, const int32_t* cu,
                                                      int* next, uint32_t k, const Watchdog& wd) {
  UnitInfo u{-1, 0, 0, 0, 0, 0};
  if ((threadIdx.x & 31) == 0) u = unit_produce(r, us, cu, next, k, wd);
  u.w = __shfl_sync(0xFFFFFFFFu, u.w, 0);
  u.doc = __shfl_sync(0xFFFFFFFFu, u.doc, 0);
  u.tile = __shfl_sync(0xFFFFFFFFu, u.tile, 0);
  u.h = __shfl_sync(0xFFFFFFFFu, u.h, 0);
  u.s = __shfl_sync(0xFFFFFFFFu, u.s, 0);
  u.e = __shfl_sync(0xFFFFFFFFu, u.e, 0);
  return u;
}

// Consumer, one thread (arrives once).
__device__ __forceinline__ UnitInfo unit_take(const UnitRing& r, uint32_t k, const Watchdog& wd) {
  const int slot = k % kUnitRing;
  if (!mbar_wait(r.full + slot, (k / kUnitRing) & 1, wd, 91)) return UnitInfo{-1, 0, 0, 0, 0, 0};
  const UnitInfo u = unit_read(r, slot);
  mbar_arrive(r.empty + slot);
  return u;
}

// Consumer, a whole warp (arrives once for the warp).
__device__ __forceinline__ UnitInfo unit_take_warp(const UnitRing& r, uint32_t k, const Watchdog& wd) {
  const int slot = k % kUnitRing;
  if (!__all_sync(0xFFFFFFFFu, mbar_wait(r.full + slot, (k / kUnitRing) & 1, wd, 92)))
    return UnitInfo{-1, 0, 0, 0, 0, 0};
  const UnitInfo u = unit_read(r, slot);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(r.empty + slot);
  return u;
}

}  // namespace fapk
