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

// Ring of unit indices in shared memory: one producer thread (it takes the
// next unit from the global counter), every other role consumes each entry
// once.  The entry past the last unit (index >= n_units) ends every role.
constexpr int kUnitRing = 8;

struct UnitRing {
  int* ids;         // [kUnitRing]
  uint64_t* full;   // [kUnitRing], 1 arrival (the producer)
  uint64_t* empty;  // [kUnitRing], one arrival per consumer (thread or warp)
};

__device__ __forceinline__ void unit_ring_init(const UnitRing& r, int consumers) {
  for (int i = 0; i < kUnitRing; ++i) {
    mbar_init(r.full + i, 1);
    mbar_init(r.empty + i, consumers);
  }
}

// Producer (one thread): the k-th unit of this CTA.  Returns -1 if a wait
// gave up.
__device__ __forceinline__ int unit_produce(const UnitRing& r, int* next, uint32_t k, const Watchdog& wd) {
  const int slot = k % kUnitRing;
  const uint32_t use = k / kUnitRing;
  if (use > 0 && !mbar_wait(r.empty + slot, (use - 1) & 1, wd, 90)) return -1;
  const int w = atomicAdd(next, 1);
  r.ids[slot] = w;
  mbar_arrive(r.full + slot);
  return w;
}

// Consumer, one thread (arrives once).
__device__ __forceinline__ int unit_take(const UnitRing& r, uint32_t k, const Watchdog& wd) {
  const int slot = k % kUnitRing;
  if (!mbar_wait(r.full + slot, (k / kUnitRing) & 1, wd, 91)) return -1;
  const int w = r.ids[slot];
  mbar_arrive(r.empty + slot);
  return w;
}

// Consumer, a whole warp (arrives once for the warp).
__device__ __forceinline__ int unit_take_warp(const UnitRing& r, uint32_t k, const Watchdog& wd) {
  const int slot = k % kUnitRing;
  if (!__all_sync(0xFFFFFFFFu, mbar_wait(r.full + slot, (k / kUnitRing) & 1, wd, 92))) return -1;
  const int w = r.ids[slot];
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(r.empty + slot);
  return w;
}

}  // namespace fapk
