// Workload-aware work order for packed documents (FLAMIA page, sec. "FLAMIA
// Mimarisi ve Temel Tasarim Ilkeleri": documents are processed in their packed
// layout without repacking, and the schedule is workload-aware).
//
// Documents are counting-sorted by their tile count, longest first; the
// sorted table records each document and the index of its first tile (a
// document's tiles follow those of all longer documents).  The kernels number
// their work units over this table (see unit_decode in sched.cuh) and take
// them from an atomic counter, which this kernel resets.  Documents of equal
// length land in whatever order the atomics give; every unit's computation is
// independent of which CTA runs it and when, so results are unaffected.
#include "internal.h"
#include "ptx.cuh"

namespace fapk {

__global__ void __launch_bounds__(1024) schedule_kernel(const int32_t* __restrict__ cu, int n_docs, int rows,
                                                        SchedBuf sb, DeviceStatus* status, int clear_status) {
  const int tid = threadIdx.x;
  const int L1 = sb.max_levels + 2;
  int* hist = sb.scratch;           // documents per tile count, then running positions
  int* doc_off = sb.scratch + L1;   // first sorted position of each tile count
  int* tile_off = sb.scratch + 2 * L1;  // first tile index of each tile count
  if (tid == 0) {
    if (clear_status) {
      status->code = 0;
      status->where = 0;
      status->block = 0;
    }
    *sb.next = 0;
  }
  for (int i = tid; i < L1; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int k = tid; k < n_docs; k += blockDim.x) {
    const int L = cu[k + 1] - cu[k];
    const int nt = (L + rows - 1) / rows;
    if (L < 0 || nt > sb.max_levels) {
      record_error(status, kStatusBadSeqlens, 1);
      continue;
    }
    if (nt > 0) atomicAdd(&hist[nt], 1);
  }
  __syncthreads();
  if (tid == 0) {
    // longest documents first: offsets of each tile count, counted from the top
    int docs = 0, tiles = 0;
    for (int l = sb.max_levels; l >= 1; --l) {
      const int c = hist[l];
      doc_off[l] = docs;
      tile_off[l] = tiles;
      hist[l] = docs;
      docs += c;
      tiles += c * l;
    }
    sb.counts[0] = docs;
    sb.counts[1] = tiles;
  }
  __syncthreads();
  for (int k = tid; k < n_docs; k += blockDim.x) {
    const int L = cu[k + 1] - cu[k];
    const int nt = (L + rows - 1) / rows;
    if (L <= 0 || nt > sb.max_levels) continue;
    const int pos = atomicAdd(&hist[nt], 1);
    sb.docs[pos] = make_int2(k, tile_off[nt] + (pos - doc_off[nt]) * nt);
  }
}

cudaError_t launch_schedule(const int32_t* cu, int n_docs, int rows, const SchedBuf& sb, DeviceStatus* status,
                            bool clear_status, cudaStream_t stream) {
  schedule_kernel<<<1, 1024, 0, stream>>>(cu, n_docs, rows, sb, status, clear_status ? 1 : 0);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace fapk
