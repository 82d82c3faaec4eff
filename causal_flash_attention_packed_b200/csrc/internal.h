// Internal interfaces between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "fapk.h"

namespace fapk {

// 32-byte alignment of an output buffer: kernels then write whole 32-byte
// sectors per store instruction (null counts as aligned).
inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

struct DeviceStatus;

// Optional CUDA events recorded between a call's kernel launches (profiling).
struct Marks {
  void* const* ev = nullptr;
  int n = 0;
  void at(int i, cudaStream_t s) const {
    if (ev && i < n && ev[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
  }
};

// Work order of the persistent kernels (schedule.cu).  Each document of
// length L has ceil(L / rows) tiles; a work unit is (document, head, tile).
// Units are numbered document by document (longest documents first), and
// within a document head by head, each head's tiles longest work first:
//  kSchedQ:  query tiles, last tile first (a later query tile sees more keys)
//  kSchedKV: key tiles, first tile first  (an earlier key tile is seen by
//                                          more queries)
// so the units that run side by side share their streamed K/V (or Q/dO)
// tiles through L2.  The CTAs take units in this order from an atomic
// counter, so the short units of the smallest documents come last.
enum SchedMode : int { kSchedQ = 0, kSchedKV = 1 };

// Scratch of one work order inside the workspace.
struct SchedBuf {
  int* scratch;   // [3 * (max_levels + 2)]: tile-count histogram and offsets
  int2* docs;     // [n_docs]: {document, index of its first tile}, longest first
  int* counts;    // [0] documents with at least one tile, [1] tiles in all
  int* next;      // the units handed out so far (reset by the scheduler)
  int max_levels;
  int max_items;  // upper bound of the tile count (grid sizing)
};

// What the kernels read of a work order.
struct SchedView {
  const int2* docs;
  const int* counts;
  int* next;
};

inline SchedView sched_view(const SchedBuf& b) { return SchedView{b.docs, b.counts, b.next}; }

cudaError_t launch_schedule(const int32_t* cu, int n_docs, int rows, const SchedBuf& sb, DeviceStatus* status,
                            bool clear_status, cudaStream_t stream);

// deq_pt_bf16 (optional): also write the per-token form dequantised to bf16.
cudaError_t launch_quantize_mxfp8(const void* x, int T, int H, int d, const int32_t* cu, int n_docs,
                                  int forms, int rule, uint8_t* vtb, uint8_t* stb, uint8_t* vpt,
                                  uint8_t* spt, cudaStream_t stream, void* deq_pt_bf16 = nullptr);

// One tensor of a quantisation launch: bf16 x [T][H][d] and its forms.
// padded: the forms are laid out with 128 codes and 4 scale bytes per
// (token, head) whatever d -- the layout the MXFP8 attention kernels read --
// so that for d = 64 channels 64..127 hold zero codes (scale byte 127): an
// all-zero 32-channel group contributes nothing to any product and leaves
// the real groups' scales alone.
struct QuantJob {
  const __nv_bfloat16* x;
  int H;
  uint8_t *vtb, *stb, *vpt, *spt;
  __nv_bfloat16* deq;  // per-token form dequantised to bf16, or null
  bool padded;
  // NVFP4 form (d = 128 only), or null: codes [T][H][64], scales [T][H][8],
  // decode scale g (six_g = fp32(6 g))
  uint8_t* nvv = nullptr;
  uint8_t* nvs = nullptr;
  float nv_g = 1.f, nv_six_g = 6.f;
};
struct QuantJobs {
  QuantJob job[2];
};
// D_i = dO_i . (o_i + o_resid_i), fp32 [Hq][T], computed by the quantisation
// launch of dO (x = dO) in the same pass.
struct DeltaArgs {
  const __nv_bfloat16* o = nullptr;
  const __nv_bfloat16* o_resid = nullptr;
  float* delta = nullptr;
  int T = 0;
};
// Up to two tensors of the same T and d in one launch (blockIdx.z = job).
cudaError_t launch_quantize_jobs(const QuantJobs& jobs, int n_jobs, int T, int d, const int32_t* cu, int n_docs,
                                 int forms, int rule, cudaStream_t stream);
// NVFP4 of a bf16 [T][H][128] tensor alone: codes [T][H][64], scales [T][H][8].
cudaError_t launch_quantize_nvfp4(const void* x, int T, int H, float g, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t stream);
// dO: both forms, and D in the same read.
cudaError_t launch_quantize_with_delta(const QuantJob& job, int T, int d, const int32_t* cu, int n_docs, int rule,
                                       const DeltaArgs& da, cudaStream_t stream);

// Per-CTA (start, end) %globaltimer records of one persistent kernel launch:
// [0] = CTA count, then one pair per CTA (kMaxCtaTimes CTAs at most).
constexpr int kMaxCtaTimes = 1024;
constexpr size_t kCtaTimesWords = 1 + 2 * (size_t)kMaxCtaTimes;

// Forward, bf16 operands (fwd_bf16.cu).
struct FwdArgs {
  unsigned long long* cta_times[2] = {nullptr, nullptr};  // per kernel, or null
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  void* o_resid;  // bf16 [T][Hq][d]: O_fp32 - bf16(O_fp32), for the backward's D
  void* v16;      // fp16 copy of V [T][Hkv][d] (the PV operand), kept for the backward
  const int32_t* cu;
  int T, Hq, Hkv, d;
  float scale;
  SchedBuf sched;
  DeviceStatus* status;
  uint64_t timeout_ns;
  int flags;
  int num_sms;
};
cudaError_t launch_fwd_bf16(const FwdArgs& a, cudaStream_t stream);

// Forward, MXFP8 path (fwd_mxfp8.cu): Q is quantised on load by the kernel
// (and its forms written to ctx); K and V codes and scales come from the
// quantiser's prepass.
struct FwdMxArgs {
  unsigned long long* cta_times[2] = {nullptr, nullptr};  // per kernel, or null
  const void* q;             // Q bf16 [T][Hq][128], quantised on load
  uint8_t* q_vpt;            // out: Q per-token codes [T][Hq][128]
  uint8_t* q_spt;            // out: Q per-token scales [T][Hq][4]
  uint8_t* q_vtb;            // out: Q token-block codes [T][Hq][128]
  uint8_t* q_stb;            // out: Q token-block scales [T/32 + n_docs][Hq][4]
  const uint8_t* k_vtb;      // K token-block codes [T][Hkv][128]
  const uint8_t* k_stb;      // K token-block scales [T/32 + n_docs][Hkv][4]
  const uint8_t* k_vpt;      // K per-token codes
  const uint8_t* k_spt;      // K per-token scales
  const uint8_t* v_vtb;      // V token-block codes
  const uint8_t* v_stb;      // V token-block scales
  const uint8_t* v_vpt;      // V per-token codes (diagonal tiles, dequantised on load)
  const uint8_t* v_spt;      // V per-token scales
  // mixed NVFP4/FP8 path (nv): the scores from NVFP4 Q (quantised on load,
  // written to q_nvv/q_nvs unless null) and K (k_nvv, k_nvs, from the prepass)
  bool nv = false;
  const uint8_t* k_nvv = nullptr;  // K NVFP4 codes [T][Hkv][64]
  const uint8_t* k_nvs = nullptr;  // K NVFP4 scales [T][Hkv][8]
  uint8_t* q_nvv = nullptr;        // out: Q NVFP4 codes [T][Hq][64]
  uint8_t* q_nvs = nullptr;        // out: Q NVFP4 scales [T][Hq][8]
  float nv_g_q = 1.f, nv_g_k = 1.f;  // decode scales
  void* o;
  float* lse;
  void* o_resid;
  const int32_t* cu;
  int T, Hq, Hkv, n_docs, d;
  float scale;
  int rule;
  SchedBuf sched;
  DeviceStatus* status;
  uint64_t timeout_ns;
  int num_sms;
};
cudaError_t launch_fwd_mxfp8(const FwdMxArgs& a, cudaStream_t stream);

// Backward, MXFP8 path (bwd_mxfp8.cu).
struct BwdMxArgs {
  unsigned long long* cta_times[2] = {nullptr, nullptr};  // per kernel, or null
  const uint8_t *q_vtb, *q_stb, *q_vpt, *q_spt;     // quantised Q (ctx)
  const uint8_t *k_vtb, *k_stb, *k_vpt, *k_spt;     // quantised K (ctx)
  const uint8_t *v_vtb, *v_stb, *v_vpt, *v_spt;     // quantised V (ctx)
  const uint8_t *do_vtb, *do_stb, *do_vpt, *do_spt; // quantised dO (workspace; written by the D pass)
  // mixed NVFP4/FP8 path (nv): the scores from the forward's NVFP4 Q and K (ctx)
  bool nv = false;
  const uint8_t *q_nvv = nullptr, *q_nvs = nullptr, *k_nvv = nullptr, *k_nvs = nullptr;
  float nv_g_q = 1.f, nv_g_k = 1.f;
  const void* o;
  const void* o_resid;
  const float* lse;
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  float* delta;
  const int32_t* cu;
  int T, Hq, Hkv, n_docs, d;
  float scale;
  int grad_bf16;
  int rule;
  SchedBuf sched_kv;
  SchedBuf sched_q;
  Marks marks;
  DeviceStatus* status;
  uint64_t timeout_ns;
  int num_sms;
};
cudaError_t launch_bwd_mxfp8(const BwdMxArgs& a, cudaStream_t stream);

// Fused QKV projection with the MX quantisation of K and V in its epilogue
// (qkv_proj.cu).  x [T][Dm] bf16, w [(Hq + 2 Hkv) 128][Dm] bf16; outputs q
// [T][Hq][128], k, v [T][Hkv][128] bf16 and K's and V's MX forms.
struct QkvProjArgs {
  const void* x;
  const void* w;
  void *q, *k, *v;
  uint8_t *k_vtb, *k_stb, *k_vpt, *k_spt;
  uint8_t *v_vtb, *v_stb, *v_vpt, *v_spt;
  // K's NVFP4 form (mixed path) instead of its MX forms, or null
  uint8_t* k_nvv = nullptr;  // codes [T][Hkv][64]
  uint8_t* k_nvs = nullptr;  // scales [T][Hkv][8]
  float nv_g_k = 1.f;        // K's decode scale
  const int32_t* cu;
  int T, Dm, Hq, Hkv;
  int rule;
  SchedBuf sched;  // 128-row tiles per document
  DeviceStatus* status;
  uint64_t timeout_ns;
  int num_sms;
};
cudaError_t launch_qkv_proj(const QkvProjArgs& a, cudaStream_t stream);

// Tensor map of E4M3 codes [T][H][128] as (128, H, T), box 128 x 1 x 128,
// 128-byte swizzle (api.cu).
bool make_tmap_codes(CUtensorMap* map, const void* base, int T, int H);
// NVFP4 codes [T][H][64 bytes]: boxes of 128 rows x 64 bytes, 64-byte swizzle.
bool make_tmap_nv(CUtensorMap* map, const void* base, int T, int H);

// Backward, bf16 operands (bwd_bf16.cu).
struct BwdArgs {
  unsigned long long* cta_times[2] = {nullptr, nullptr};  // per kernel, or null
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const float* lse;
  const void* dout;
  const void* o_resid;  // residual of O written by the forward
  const void* v16;      // fp16 V written by the forward
  void* q16;            // fp16 copies made by the backward's prepass ([T][Hq][d], [T][Hkv][d], [T][Hq][d])
  void* k16;
  void* do16;
  void* dq;
  void* dk;
  void* dv;
  float* delta;  // [Hq][T] fp32 scratch: D_i = dO_i . O_i
  float* nl2;    // [Hq][T] fp32 scratch: -LSE_i log2(e)
  const int32_t* cu;
  int T, Hq, Hkv, d;
  float scale;
  int grad_bf16;
  SchedBuf sched_kv;
  SchedBuf sched_q;
  Marks marks;  // [3] before D, [4] before dK/dV, [5] before dQ, [6] after
  DeviceStatus* status;
  uint64_t timeout_ns;
  int flags;
  int num_sms;
};
cudaError_t launch_bwd_bf16(const BwdArgs& a, cudaStream_t stream);

// Tensor map of a 16-bit [T][H][d] tensor (bf16, or fp16 when `f16`) as a 3-D
// (d, H, T) view with a box of 64 channels x 1 head x 128 tokens and 128-byte
// swizzle (api.cu).
// Tensor map of a [T][H][d] 16-bit tensor: boxes of 64 channels x 1 head x
// 128 tokens, 128-byte swizzle.
bool make_tmap_thd(CUtensorMap* map, const void* base, int T, int H, int d, bool f16 = false);

// bf16 -> fp16 copy of n elements (n a multiple of 8); magnitudes >= 65504
// record kStatusRange (convert.cu).
cudaError_t launch_convert_f16(const void* src, void* dst, long long n, DeviceStatus* status, int num_sms,
                               cudaStream_t stream);

// Count of kernels launched by this library (api.cu).
void note_launches(int n);

}  // namespace fapk
