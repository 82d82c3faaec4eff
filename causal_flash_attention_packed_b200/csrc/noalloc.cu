// Forward entry point that allocates nothing (fapk_attn_fwd_noalloc).
//
// Some callers cannot obtain device memory at the point where they run the
// forward: a plugin that is handed its input and output buffers by a host
// framework and must not allocate behind its back, or an embedded runtime
// that reserves all device memory at start-up.  For them the forward's
// scratch (the device status word and the scheduler's work list) lives in a
// fixed array compiled into the library.  Inputs, outputs and the saved-state
// buffer ctx are still the caller's.  These entry points make CUDA runtime
// calls (device query, symbol lookup, kernel launches), so, like any CUDA
// call, they must not be made from inside a stream callback
// (cudaLaunchHostFunc / cudaStreamAddCallback).
//
// The array is file-scope device memory: every GPU that loads the library
// holds its kNoAllocScratchBytes until the process exits.  With CUDA's lazy
// module loading (the default) that memory is taken when this file's module
// is first loaded on a device, which happens at the first cudaGetSymbolAddress
// below, i.e. during the first call on that device: make that first call
// before reserving the rest of the device's memory, and before any stream
// capture.  Host code may not hand the array's name to a kernel (on the host
// that name is only a stand-in, not a device address); the device address is
// looked up once per device with cudaGetSymbolAddress, with that device
// current, and cached.  Every call shares the one array and leaves its
// contents behind; the forward's scheduler clears the status word and its
// counters at the start of each call, and calls whose GPU work overlaps (other
// streams, other host threads) race on the array.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB

static __device__ __align__(256) unsigned char g_fwd_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_fwd_scratch on the current device (nullptr on error).
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_fwd_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

int fapk_attn_fwd_noalloc(const fapk_problem_t* prob, const void* q, const void* k, const void* v, void* o,
                          float* lse, void* ctx, void* stream) {
  if (!prob) return FAPK_ERR_INVALID_ARG;
  if (prob->T > 0) {
    const size_t need = fapk_workspace_size(prob, FAPK_FWD);
    // an invalid problem: let the regular entry point report the exact code
    if (need == 0) return fapk_attn_fwd(prob, q, k, v, o, lse, ctx, nullptr, 0, stream);
    if (need > kNoAllocScratchBytes) return FAPK_ERR_WORKSPACE_TOO_SMALL;
  }
  void* ws = scratch_address();
  if (!ws) return FAPK_ERR_CUDA;
  return fapk_attn_fwd(prob, q, k, v, o, lse, ctx, ws, kNoAllocScratchBytes, stream);
}

int fapk_noalloc_status(void* stream) {
  void* ws = scratch_address();
  if (!ws) return FAPK_ERR_CUDA;
  // the status word sits at the start of the forward's workspace
  return fapk_status(ws, stream);
}

}  // extern "C"
