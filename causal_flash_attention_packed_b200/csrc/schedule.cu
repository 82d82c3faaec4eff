// Workload-aware scheduling of packed documents (FLAMIA page, sec. "FLAMIA
// Mimarisi ve Temel Tasarim Ilkeleri": documents are processed in their packed
// layout without repacking, and the schedule is workload-aware).
//
// Each document of length L contributes ceil(L / rows) tiles.  The work of a
// tile under the causal mask grows with its query index (or, for key tiles,
// with the number of later query tiles), so tiles are bucketed by a cost level
// and emitted highest level first: persistent CTAs that take items in list
// order get the longest work first (longest-processing-time-first balancing).
// Within one level the order is whatever the atomics give; every item's
// computation is independent of which CTA runs it, so results are unaffected.
#include "internal.h"
#include "ptx.cuh"

namespace fapk {

__global__ void __launch_bounds__(1024) schedule_kernel(const int32_t* __restrict__ cu, int n_docs,
                                                        int rows, int mode, SchedBuf sb,
                                                        DeviceStatus* status, int clear_status) {
  const int tid = threadIdx.x;
  int* off = sb.level_off;  // histogram, then running level offsets
  if (tid == 0 && clear_status) {
    status->code = 0;
    status->where = 0;
    status->block = 0;
  }
  for (int i = tid; i < sb.max_levels + 2; i += blockDim.x) off[i] = 0;
  __syncthreads();
  // histogram of tiles per document: off[nt] += 1
  for (int k = tid; k < n_docs; k += blockDim.x) {
    const int L = cu[k + 1] - cu[k];
    const int nt = (L + rows - 1) / rows;
    if (L < 0 || nt > sb.max_levels) {
      record_error(status, kStatusBadSeqlens, 1);
      continue;
    }
    if (nt > 0) atomicAdd(&off[nt], 1);
  }
  __syncthreads();
  if (tid == 0) {
    // count[l] = number of documents with more than l tiles = sum_{n > l} hist[n];
    // levels are emitted highest first: offset[l] = sum_{l' > l} count[l'].
    int suffix = 0;  // running count[l]
    int total = 0;   // items of levels above l
    for (int l = sb.max_levels; l >= 1; --l) {
      suffix += off[l];  // documents with exactly l tiles join count[l - 1]
      const int c = suffix;
      off[l] = total;    // reuse slot l as the offset of level l - 1
      total += c;
    }
    off[0] = 0;
    *sb.n_items = total;
  }
  __syncthreads();
  // place: level lvl's offset sits in off[lvl + 1]
  for (int k = tid; k < n_docs; k += blockDim.x) {
    const int L = cu[k + 1] - cu[k];
    const int nt = (L + rows - 1) / rows;
    if (L <= 0 || nt > sb.max_levels) continue;
    for (int t = 0; t < nt; ++t) {
      const int lvl = (mode == kSchedQ) ? t : (nt - 1 - t);
      const int pos = atomicAdd(&off[lvl + 1], 1);
      if (pos < sb.max_items) sb.list[pos] = make_int2(k, t);
    }
  }
}

cudaError_t launch_schedule(const int32_t* cu, int n_docs, int rows, int mode, const SchedBuf& sb,
                            DeviceStatus* status, bool clear_status, cudaStream_t stream) {
  schedule_kernel<<<1, 1024, 0, stream>>>(cu, n_docs, rows, mode, sb, status, clear_status ? 1 : 0);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace fapk
