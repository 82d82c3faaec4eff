// C-ABI entry points of fapk (declared in include/fapk.h): argument
// validation on the host, workspace layout, TMA descriptor creation and the
// kernel launches.  No entry point allocates device memory or synchronises,
// except fapk_status.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace fapk {

namespace {

std::atomic<uint64_t> g_launches{0};

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// --- driver entry point for tensor-map encoding (no libcuda link needed) ---
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// --- per-device cached attributes ---
constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int g_num_sms[kMaxDevices] = {0};

int device_num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_num_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// --- problem validation ---
// The MXFP8 machinery (quantised forms in ctx, the MX kernels) serves both
// low-precision paths.
bool is_mx(const fapk_problem_t* P) { return P->prec == FAPK_MXFP8 || P->prec == FAPK_NVFP4_MIXED; }
// An NVFP4 decode scale: 0 (selects 1) or a finite value in [2^-100, 2^100],
// so that no step of the quantisation overflows fp32.
bool nv_scale_ok(float g) { return g == 0.f || (std::isfinite(g) && g >= 0x1p-100f && g <= 0x1p100f); }
float nv_scale_of(float g) { return g == 0.f ? 1.f : g; }

int validate_problem(const fapk_problem_t* P) {
  if (!P) return FAPK_ERR_INVALID_ARG;
  if (P->T < 0 || P->n_docs < 0 || P->Hq <= 0 || P->Hkv <= 0) return FAPK_ERR_INVALID_ARG;
  if (P->d != 64 && P->d != 128) return FAPK_ERR_UNSUPPORTED;
  if (P->Hq % P->Hkv != 0) return FAPK_ERR_UNSUPPORTED;
  if (P->prec != FAPK_BF16 && P->prec != FAPK_MXFP8 && P->prec != FAPK_NVFP4_MIXED) return FAPK_ERR_UNSUPPORTED;
  if (P->scale_rule != FAPK_SCALE_RCEIL && P->scale_rule != FAPK_SCALE_OCP) return FAPK_ERR_UNSUPPORTED;
  // the attention path quantises with RCEIL only: under OCP the computed
  // operands quantise discontinuously near powers of two (see fapk.h)
  if (is_mx(P) && P->scale_rule != FAPK_SCALE_RCEIL) return FAPK_ERR_UNSUPPORTED;
  if (P->prec == FAPK_NVFP4_MIXED) {
    if (!nv_scale_ok(P->nv_scale_q) || !nv_scale_ok(P->nv_scale_k)) return FAPK_ERR_INVALID_ARG;
  }
  if (P->grad_dtype != FAPK_GRAD_F32 && P->grad_dtype != FAPK_GRAD_BF16) return FAPK_ERR_UNSUPPORTED;
  if (!std::isfinite(P->scale)) return FAPK_ERR_INVALID_ARG;
  if (P->T > 0) {
    if (P->n_docs < 1 || P->max_seqlen < 1 || !P->cu_seqlens_dev) return FAPK_ERR_INVALID_ARG;
    // 64-bit element offsets are used everywhere; keep token and head counts
    // inside what the TMA coordinates (int32) and grid dimensions allow
    if ((long long)P->T * P->Hq * P->d > (1LL << 40)) return FAPK_ERR_UNSUPPORTED;
  }
  if (P->cu_seqlens_host) {
    const int32_t* cu = P->cu_seqlens_host;
    if (cu[0] != 0 || cu[P->n_docs] != P->T) return FAPK_ERR_BAD_SEQLENS;
    for (int k = 0; k < P->n_docs; ++k) {
      const int L = cu[k + 1] - cu[k];
      if (L < 0 || L > P->max_seqlen) return FAPK_ERR_BAD_SEQLENS;
    }
  }
  return FAPK_OK;
}

uint64_t timeout_ns_of(const fapk_problem_t* P) {
  const int ms = P->timeout_ms > 0 ? P->timeout_ms : 2000;
  return (uint64_t)ms * 1000000ull;
}

// --- workspace layout ---
struct SchedLayout {
  size_t scratch, docs, counts, next, end;
  int max_levels, max_items;
};

SchedLayout sched_layout(size_t base, int T, int n_docs, int max_seqlen, int rows) {
  SchedLayout s;
  s.max_levels = (max_seqlen + rows - 1) / rows;
  s.max_items = T / rows + n_docs + 1;
  s.scratch = align_up(base);
  s.docs = align_up(s.scratch + sizeof(int) * 3 * (size_t)(s.max_levels + 2));
  s.counts = align_up(s.docs + sizeof(int2) * (size_t)(n_docs > 0 ? n_docs : 1));
  s.next = align_up(s.counts + 2 * sizeof(int));
  s.end = align_up(s.next + sizeof(int));
  return s;
}

SchedBuf sched_buf(void* ws, const SchedLayout& s) {
  char* w = static_cast<char*>(ws);
  SchedBuf b;
  b.scratch = reinterpret_cast<int*>(w + s.scratch);
  b.docs = reinterpret_cast<int2*>(w + s.docs);
  b.counts = reinterpret_cast<int*>(w + s.counts);
  b.next = reinterpret_cast<int*>(w + s.next);
  b.max_levels = s.max_levels;
  b.max_items = s.max_items;
  return b;
}

constexpr int kFwdRows = 256;  // query rows per forward work item (two 128-row tiles)
constexpr int kBwdRows = 128;  // rows per backward work item

constexpr int kFwdRowsMx = 128;  // query rows per MXFP8 forward work item (one tile)

struct FwdLayout {
  SchedLayout sched;
  size_t cta_times, total;
};
FwdLayout fwd_layout(const fapk_problem_t* P) {
  FwdLayout L;
  L.sched = sched_layout(kAlign, P->T, P->n_docs, P->max_seqlen,
                         is_mx(P) ? kFwdRowsMx : kFwdRows);
  L.cta_times = align_up(L.sched.end);
  L.total = align_up(L.cta_times + sizeof(unsigned long long) * kCtaTimesWords);
  return L;
}

// Backward workspace: two work lists, D = rowsum(dO * O) in fp32 and the fp16
// copies of Q, K and dO that the gradient MMAs read.
//  MXFP8 path, instead of the fp16 copies: the quantiser's forms of dO.
struct BwdLayout {
  SchedLayout kv, q;
  size_t delta, q16, k16, do16, nl2, cta_times, total;
  size_t do_vtb, do_stb, do_vpt, do_spt;
};
BwdLayout bwd_layout(const fapk_problem_t* P) {
  BwdLayout L;
  const size_t nq = (size_t)P->T * P->Hq * P->d, nk = (size_t)P->T * P->Hkv * P->d;
  L.kv = sched_layout(kAlign, P->T, P->n_docs, P->max_seqlen, kBwdRows);
  L.q = sched_layout(L.kv.end, P->T, P->n_docs, P->max_seqlen, kBwdRows);
  L.delta = L.q.end;
  const size_t after_delta = align_up(L.delta + sizeof(float) * (size_t)P->Hq * (size_t)P->T);
  if (is_mx(P)) {
    const size_t slots = (size_t)P->T / 32 + P->n_docs;
    L.q16 = L.k16 = L.do16 = 0;
    // dO's MX forms, 128 codes and 4 scale bytes per (token, head) for any d
    const size_t nq128 = (size_t)P->T * P->Hq * 128;
    L.do_vtb = after_delta;
    L.do_stb = align_up(L.do_vtb + nq128);
    L.do_vpt = align_up(L.do_stb + slots * P->Hq * 4);
    L.do_spt = align_up(L.do_vpt + nq128);
    L.cta_times = align_up(L.do_spt + (size_t)P->T * P->Hq * 4);
    L.total = align_up(L.cta_times + 2 * sizeof(unsigned long long) * kCtaTimesWords);
    return L;
  }
  L.q16 = after_delta;
  L.k16 = align_up(L.q16 + 2 * nq);
  L.do16 = align_up(L.k16 + 2 * nk);
  L.nl2 = align_up(L.do16 + 2 * nq);
  L.cta_times = align_up(L.nl2 + sizeof(float) * (size_t)P->Hq * (size_t)P->T);
  L.total = align_up(L.cta_times + 2 * sizeof(unsigned long long) * kCtaTimesWords);
  return L;
}

// Saved state from the forward to the backward (the caller's ctx buffer):
//  o_resid: bf16 [T][Hq][d], O_fp32 - bf16(O_fp32), so that the backward's
//           D_i = dO_i . O_i uses O to about 16 significant bits rather than
//           the 8 of the bf16 output;
//  v16:     fp16 copy of V [T][Hkv][d], the B operand of O += P V (and of the
//           backward's dP = dO V^T).
//  MXFP8 path, instead of v16: the MX forms of Q, K and V (codes and scales,
//  token-block and per-token), reused by the backward in both orientations;
//  Q's are written by the forward kernel, which quantises Q on load, K's and
//  V's by the quantiser's prepass.
struct MxForms {
  size_t vtb, stb, vpt, spt;  // offsets of codes / scales
};
struct CtxLayout {
  size_t o_resid, v16, total;
  MxForms q, k, v;
  // mixed NVFP4/FP8 path: NVFP4 codes [T][H][64] and scales [T][H][8] of Q and K
  size_t q_nvv = 0, q_nvs = 0, k_nvv = 0, k_nvs = 0;
};
CtxLayout ctx_layout(const fapk_problem_t* P) {
  CtxLayout L;
  L.o_resid = 0;
  size_t off = align_up(sizeof(uint16_t) * (size_t)P->T * P->Hq * P->d);
  if (!is_mx(P)) {
    L.v16 = off;
    L.total = align_up(L.v16 + sizeof(uint16_t) * (size_t)P->T * P->Hkv * P->d);
    return L;
  }
  L.v16 = 0;
  const size_t slots = (size_t)P->T / 32 + P->n_docs;
  // 128 codes and 4 scale bytes per (token, head) for any d (d = 64: the
  // upper half holds zero codes)
  auto forms = [&](int H) {
    MxForms f;
    const size_t n = (size_t)P->T * H * 128;
    f.vtb = off;
    f.stb = align_up(f.vtb + n);
    f.vpt = align_up(f.stb + slots * H * 4);
    f.spt = align_up(f.vpt + n);
    off = align_up(f.spt + (size_t)P->T * H * 4);
    return f;
  };
  L.q = forms(P->Hq);
  L.k = forms(P->Hkv);
  L.v = forms(P->Hkv);
  if (P->prec == FAPK_NVFP4_MIXED) {
    L.q_nvv = off;
    L.q_nvs = align_up(L.q_nvv + (size_t)P->T * P->Hq * 64);
    L.k_nvv = align_up(L.q_nvs + (size_t)P->T * P->Hq * 8);
    L.k_nvs = align_up(L.k_nvv + (size_t)P->T * P->Hkv * 64);
    off = align_up(L.k_nvs + (size_t)P->T * P->Hkv * 8);
  }
  L.total = off;
  return L;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? FAPK_OK : FAPK_ERR_CUDA; }

}  // namespace

void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

bool make_tmap_codes(CUtensorMap* map, const void* base, int T, int H) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {128, (cuuint64_t)H * 128};
  const cuuint32_t box[3] = {128, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_nv(CUtensorMap* map, const void* base, int T, int H) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {64, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {64, (cuuint64_t)H * 64};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_thd(CUtensorMap* map, const void* base, int T, int H, int d, bool f16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// MXFP8 forward: build the 128-row schedule, quantise K and V into ctx (both
// forms, one launch), run the kernel (which quantises Q on load and writes its
// forms into ctx).
int fwd_mxfp8(const fapk_problem_t* P, const void* q, const void* k, const void* v, void* o, float* lse, void* ctx,
              void* ws, const FwdLayout& L, int sms, cudaStream_t st) {
  auto* status = static_cast<DeviceStatus*>(ws);
  const CtxLayout C = ctx_layout(P);
  char* c = static_cast<char*>(ctx);
  auto u8 = [&](size_t off) { return reinterpret_cast<uint8_t*>(c + off); };
  const Marks mk{P->timing_events, P->n_timing_events};
  FwdMxArgs a;
  a.sched = sched_buf(ws, L.sched);
  mk.at(0, st);
  int rc = cuda_status(launch_schedule(P->cu_seqlens_dev, P->n_docs, kFwdRowsMx, a.sched, status, true, st));
  if (rc != FAPK_OK) return rc;
  mk.at(1, st);
  QuantJobs jobs;
  jobs.job[0] = QuantJob{static_cast<const __nv_bfloat16*>(k), P->Hkv, u8(C.k.vtb), u8(C.k.stb), u8(C.k.vpt),
                         u8(C.k.spt), nullptr, true};
  jobs.job[1] = QuantJob{static_cast<const __nv_bfloat16*>(v), P->Hkv, u8(C.v.vtb), u8(C.v.stb), u8(C.v.vpt),
                         u8(C.v.spt), nullptr, true};
  const bool nv = P->prec == FAPK_NVFP4_MIXED;
  if (nv) {
    // K's NVFP4 form for the scores, in the same pass
    jobs.job[0].nvv = u8(C.k_nvv);
    jobs.job[0].nvs = u8(C.k_nvs);
    jobs.job[0].nv_g = nv_scale_of(P->nv_scale_k);
    jobs.job[0].nv_six_g = 6.0f * jobs.job[0].nv_g;
    a.nv = true;
    a.k_nvv = u8(C.k_nvv);
    a.k_nvs = u8(C.k_nvs);
    a.q_nvv = u8(C.q_nvv);
    a.q_nvs = u8(C.q_nvs);
    a.nv_g_q = nv_scale_of(P->nv_scale_q);
    a.nv_g_k = nv_scale_of(P->nv_scale_k);
  }
  rc = cuda_status(launch_quantize_jobs(jobs, 2, P->T, P->d, P->cu_seqlens_dev, P->n_docs,
                                        FAPK_FORM_TB | FAPK_FORM_PT, P->scale_rule, st));
  if (rc != FAPK_OK) return rc;
  a.q = q;
  a.q_vpt = u8(C.q.vpt);
  a.q_spt = u8(C.q.spt);
  a.q_vtb = u8(C.q.vtb);
  a.q_stb = u8(C.q.stb);
  a.k_vtb = u8(C.k.vtb);
  a.k_stb = u8(C.k.stb);
  a.k_vpt = u8(C.k.vpt);
  a.k_spt = u8(C.k.spt);
  a.v_vtb = u8(C.v.vtb);
  a.v_stb = u8(C.v.stb);
  a.v_vpt = u8(C.v.vpt);
  a.v_spt = u8(C.v.spt);
  a.o = o;
  a.lse = lse;
  a.o_resid = c + C.o_resid;
  a.cu = P->cu_seqlens_dev;
  a.T = P->T;
  a.Hq = P->Hq;
  a.Hkv = P->Hkv;
  a.n_docs = P->n_docs;
  a.d = P->d;
  a.scale = P->scale;
  a.rule = P->scale_rule;
  a.status = status;
  if (P->flags & FAPK_FLAG_CTA_TIMES)
    a.cta_times[0] = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + L.cta_times);
  a.timeout_ns = timeout_ns_of(P);
  a.num_sms = sms;
  mk.at(2, st);
  rc = cuda_status(launch_fwd_mxfp8(a, st));
  mk.at(3, st);
  return rc;
}

// MXFP8 backward: build both schedules, then D together with dO's two MX
// forms (one pass over dO, into the workspace), dK/dV and dQ.
int bwd_mxfp8(const fapk_problem_t* P, const void* o, const float* lse, const void* dout, const void* ctx, void* dq,
              void* dk, void* dv, void* ws, const BwdLayout& L, int sms, cudaStream_t st) {
  auto* status = static_cast<DeviceStatus*>(ws);
  const CtxLayout C = ctx_layout(P);
  const char* c = static_cast<const char*>(ctx);
  char* w = static_cast<char*>(ws);
  auto cu8 = [&](size_t off) { return reinterpret_cast<const uint8_t*>(c + off); };
  auto wu8 = [&](size_t off) { return reinterpret_cast<uint8_t*>(w + off); };
  BwdMxArgs a;
  a.marks = Marks{P->timing_events, P->n_timing_events};
  a.sched_kv = sched_buf(ws, L.kv);
  a.sched_q = sched_buf(ws, L.q);
  a.marks.at(0, st);
  int rc = cuda_status(launch_schedule(P->cu_seqlens_dev, P->n_docs, kBwdRows, a.sched_kv, status, true, st));
  if (rc != FAPK_OK) return rc;
  a.marks.at(1, st);
  rc = cuda_status(launch_schedule(P->cu_seqlens_dev, P->n_docs, kBwdRows, a.sched_q, status, false, st));
  if (rc != FAPK_OK) return rc;
  a.q_vtb = cu8(C.q.vtb); a.q_stb = cu8(C.q.stb); a.q_vpt = cu8(C.q.vpt); a.q_spt = cu8(C.q.spt);
  a.k_vtb = cu8(C.k.vtb); a.k_stb = cu8(C.k.stb); a.k_vpt = cu8(C.k.vpt); a.k_spt = cu8(C.k.spt);
  a.v_vtb = cu8(C.v.vtb); a.v_stb = cu8(C.v.stb); a.v_vpt = cu8(C.v.vpt); a.v_spt = cu8(C.v.spt);
  a.do_vtb = wu8(L.do_vtb); a.do_stb = wu8(L.do_stb); a.do_vpt = wu8(L.do_vpt); a.do_spt = wu8(L.do_spt);
  if (P->prec == FAPK_NVFP4_MIXED) {
    a.nv = true;
    a.q_nvv = cu8(C.q_nvv); a.q_nvs = cu8(C.q_nvs); a.k_nvv = cu8(C.k_nvv); a.k_nvs = cu8(C.k_nvs);
    a.nv_g_q = nv_scale_of(P->nv_scale_q);
    a.nv_g_k = nv_scale_of(P->nv_scale_k);
  }
  a.o = o;
  a.o_resid = c + C.o_resid;
  a.lse = lse;
  a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.delta = reinterpret_cast<float*>(w + L.delta);
  a.cu = P->cu_seqlens_dev;
  a.T = P->T; a.Hq = P->Hq; a.Hkv = P->Hkv; a.n_docs = P->n_docs; a.d = P->d;
  a.scale = P->scale;
  a.grad_bf16 = P->grad_dtype == FAPK_GRAD_BF16;
  a.rule = P->scale_rule;
  a.status = status;
  if (P->flags & FAPK_FLAG_CTA_TIMES) {
    auto* ct = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + L.cta_times);
    a.cta_times[0] = ct;
    a.cta_times[1] = ct + kCtaTimesWords;
  }
  a.timeout_ns = timeout_ns_of(P);
  a.num_sms = sms;
  return cuda_status(launch_bwd_mxfp8(a, st));
}


// The forward over pre-quantised K and V (no quantisation launch, no saved
// state): a carries K's forms (MX, or NVFP4 with a.nv); V's MX forms are
// checked and set here.
int fwd_quantized_kv(const fapk_problem_t* P, const void* q, FwdMxArgs& a, const uint8_t* v_val_tb,
                     const uint8_t* v_scale_tb, const uint8_t* v_val_pt, const uint8_t* v_scale_pt, void* o,
                     float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!q || !v_val_tb || !v_scale_tb || !v_val_pt || !v_scale_pt || !o || !lse || !ws) return FAPK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse) || !aligned16(v_val_tb) || !aligned16(v_val_pt) ||
      (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)))
    return FAPK_ERR_INVALID_ARG;
  // scale rows are read 4 bytes at a time
  for (const uint8_t* sp : {v_scale_tb, v_scale_pt})
    if (reinterpret_cast<uintptr_t>(sp) & 3u) return FAPK_ERR_INVALID_ARG;
  const FwdLayout L = fwd_layout(P);
  if (ws_bytes < L.total) return FAPK_ERR_WORKSPACE_TOO_SMALL;
  const int sms = device_num_sms();
  if (sms <= 0) return FAPK_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* status = static_cast<DeviceStatus*>(ws);
  const Marks mk{P->timing_events, P->n_timing_events};
  a.sched = sched_buf(ws, L.sched);
  mk.at(0, st);
  int rc = cuda_status(launch_schedule(P->cu_seqlens_dev, P->n_docs, kFwdRowsMx, a.sched, status, true, st));
  if (rc != FAPK_OK) return rc;
  a.q = q;
  a.q_vpt = a.q_spt = a.q_vtb = a.q_stb = nullptr;  // no saved state: nothing for a backward
  a.q_nvv = a.q_nvs = nullptr;
  a.v_vtb = v_val_tb; a.v_stb = v_scale_tb; a.v_vpt = v_val_pt; a.v_spt = v_scale_pt;
  a.o = o;
  a.lse = lse;
  a.o_resid = nullptr;
  a.cu = P->cu_seqlens_dev;
  a.T = P->T; a.Hq = P->Hq; a.Hkv = P->Hkv; a.n_docs = P->n_docs; a.d = P->d;
  a.scale = P->scale;
  a.rule = P->scale_rule;
  a.status = status;
  if (P->flags & FAPK_FLAG_CTA_TIMES)
    a.cta_times[0] = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + L.cta_times);
  a.timeout_ns = timeout_ns_of(P);
  a.num_sms = sms;
  mk.at(1, st);
  rc = cuda_status(launch_fwd_mxfp8(a, st));
  mk.at(2, st);
  return rc;
}


// The fused QKV projection: a carries K's output forms (MX, or NVFP4 when
// a.k_nvv is set); the rest is checked and set here.
int qkv_proj(const fapk_problem_t* P, const void* x, int d_model, const void* w, void* q, void* k, void* v,
             QkvProjArgs& a, uint8_t* v_val_tb, uint8_t* v_scale_tb, uint8_t* v_val_pt, uint8_t* v_scale_pt,
             void* ws, size_t ws_bytes, void* stream) {
  if (d_model <= 0 || d_model % 8 != 0) return FAPK_ERR_INVALID_ARG;
  if (P->T == 0) return FAPK_OK;
  if (!x || !w || !q || !k || !v || !v_val_tb || !v_scale_tb || !v_val_pt || !v_scale_pt || !ws)
    return FAPK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(v_val_tb) ||
      !aligned16(v_val_pt) || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)))
    return FAPK_ERR_INVALID_ARG;
  // 64-bit offsets throughout; keep the weight rows inside the TMA coordinate range
  if ((long long)(P->Hq + 2 * P->Hkv) * 128 > 0x7FFFFFFFLL) return FAPK_ERR_UNSUPPORTED;
  const FwdLayout L = fwd_layout(P);  // the MX forward's work order: 128-row tiles per document
  if (ws_bytes < L.total) return FAPK_ERR_WORKSPACE_TOO_SMALL;
  const int sms = device_num_sms();
  if (sms <= 0) return FAPK_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* status = static_cast<DeviceStatus*>(ws);
  a.sched = sched_buf(ws, L.sched);
  const Marks mk{P->timing_events, P->n_timing_events};
  mk.at(0, st);
  int rc = cuda_status(launch_schedule(P->cu_seqlens_dev, P->n_docs, kFwdRowsMx, a.sched, status, true, st));
  if (rc != FAPK_OK) return rc;
  a.x = x; a.w = w; a.q = q; a.k = k; a.v = v;
  a.v_vtb = v_val_tb; a.v_stb = v_scale_tb; a.v_vpt = v_val_pt; a.v_spt = v_scale_pt;
  a.cu = P->cu_seqlens_dev;
  a.T = P->T; a.Dm = d_model; a.Hq = P->Hq; a.Hkv = P->Hkv;
  a.rule = P->scale_rule;
  a.status = status;
  a.timeout_ns = timeout_ns_of(P);
  a.num_sms = sms;
  mk.at(1, st);
  rc = cuda_status(launch_qkv_proj(a, st));
  mk.at(2, st);
  return rc;
}

}  // namespace

}  // namespace fapk

using namespace fapk;

extern "C" {

size_t fapk_workspace_size(const fapk_problem_t* prob, int which) {
  if (validate_problem(prob) != FAPK_OK) return 0;
  if (which == FAPK_FWD) return fwd_layout(prob).total;
  if (which == FAPK_BWD) return bwd_layout(prob).total;
  return 0;
}

size_t fapk_ctx_size(const fapk_problem_t* prob) {
  if (validate_problem(prob) != FAPK_OK) return 0;
  return ctx_layout(prob).total;
}

int fapk_attn_fwd(const fapk_problem_t* P, const void* q, const void* k, const void* v, void* o,
                  float* lse, void* ctx, void* ws, size_t ws_bytes, void* stream) {
  int rc = validate_problem(P);
  if (rc != FAPK_OK) return rc;
  if (P->T == 0) return FAPK_OK;
  if (!q || !k || !v || !o || !lse || !ctx || !ws) return FAPK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(ctx) || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)))
    return FAPK_ERR_INVALID_ARG;
  const FwdLayout L = fwd_layout(P);
  if (ws_bytes < L.total) return FAPK_ERR_WORKSPACE_TOO_SMALL;
  const int sms = device_num_sms();
  if (sms <= 0) return FAPK_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* status = static_cast<DeviceStatus*>(ws);
  if (is_mx(P)) return fwd_mxfp8(P, q, k, v, o, lse, ctx, ws, L, sms, st);
  FwdArgs a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  const CtxLayout CL = ctx_layout(P);
  a.o_resid = static_cast<char*>(ctx) + CL.o_resid;
  a.v16 = static_cast<char*>(ctx) + CL.v16;
  a.cu = P->cu_seqlens_dev;
  a.T = P->T; a.Hq = P->Hq; a.Hkv = P->Hkv; a.d = P->d;
  a.scale = P->scale;
  a.sched = sched_buf(ws, L.sched);
  a.status = status;
  if (P->flags & FAPK_FLAG_CTA_TIMES)
    a.cta_times[0] = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + L.cta_times);
  a.timeout_ns = timeout_ns_of(P);
  a.flags = P->flags;
  a.num_sms = sms;
  const Marks mk{P->timing_events, P->n_timing_events};
  mk.at(0, st);
  rc = cuda_status(launch_schedule(P->cu_seqlens_dev, P->n_docs, kFwdRows, a.sched, status, true, st));
  if (rc != FAPK_OK) return rc;
  mk.at(1, st);
  rc = cuda_status(launch_convert_f16(v, a.v16, (long long)P->T * P->Hkv * P->d, status, sms, st));
  if (rc != FAPK_OK) return rc;
  mk.at(2, st);
  rc = cuda_status(launch_fwd_bf16(a, st));
  mk.at(3, st);
  return rc;
}

int fapk_attn_bwd(const fapk_problem_t* P, const void* q, const void* k, const void* v, const void* o,
                  const float* lse, const void* dout, const void* ctx, void* dq, void* dk, void* dv,
                  void* ws, size_t ws_bytes, void* stream) {
  int rc = validate_problem(P);
  if (rc != FAPK_OK) return rc;
  if (P->T == 0) return FAPK_OK;
  if (!q || !k || !v || !o || !lse || !dout || !ctx || !dq || !dk || !dv || !ws) return FAPK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(ctx) ||
      (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)))
    return FAPK_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(P);
  if (ws_bytes < L.total) return FAPK_ERR_WORKSPACE_TOO_SMALL;
  const int sms = device_num_sms();
  if (sms <= 0) return FAPK_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (is_mx(P)) return bwd_mxfp8(P, o, lse, dout, ctx, dq, dk, dv, ws, L, sms, st);
  auto* status = static_cast<DeviceStatus*>(ws);
  BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse; a.dout = dout;
  const CtxLayout CL = ctx_layout(P);
  a.o_resid = static_cast<const char*>(ctx) + CL.o_resid;
  a.v16 = static_cast<const char*>(ctx) + CL.v16;
  a.q16 = static_cast<char*>(ws) + L.q16;
  a.k16 = static_cast<char*>(ws) + L.k16;
  a.do16 = static_cast<char*>(ws) + L.do16;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.delta = reinterpret_cast<float*>(static_cast<char*>(ws) + L.delta);
  a.nl2 = reinterpret_cast<float*>(static_cast<char*>(ws) + L.nl2);
  a.cu = P->cu_seqlens_dev;
  a.T = P->T; a.Hq = P->Hq; a.Hkv = P->Hkv; a.d = P->d;
  a.scale = P->scale;
  a.grad_bf16 = P->grad_dtype == FAPK_GRAD_BF16;
  a.sched_kv = sched_buf(ws, L.kv);
  a.sched_q = sched_buf(ws, L.q);
  a.status = status;
  if (P->flags & FAPK_FLAG_CTA_TIMES) {
    auto* ct = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + L.cta_times);
    a.cta_times[0] = ct;
    a.cta_times[1] = ct + kCtaTimesWords;
  }
  a.timeout_ns = timeout_ns_of(P);
  a.flags = P->flags;
  a.num_sms = sms;
  a.marks = Marks{P->timing_events, P->n_timing_events};
  a.marks.at(0, st);
  rc = cuda_status(launch_schedule(P->cu_seqlens_dev, P->n_docs, kBwdRows, a.sched_kv, status, true, st));
  if (rc != FAPK_OK) return rc;
  a.marks.at(1, st);
  rc = cuda_status(launch_schedule(P->cu_seqlens_dev, P->n_docs, kBwdRows, a.sched_q, status, false, st));
  if (rc != FAPK_OK) return rc;
  a.marks.at(2, st);
  rc = cuda_status(launch_convert_f16(k, a.k16, (long long)P->T * P->Hkv * P->d, status, sms, st));
  if (rc != FAPK_OK) return rc;
  return cuda_status(launch_bwd_bf16(a, st));
}

int fapk_attn_fwd_quantized_kv(const fapk_problem_t* P, const void* q, const uint8_t* k_val_tb,
                               const uint8_t* k_scale_tb, const uint8_t* k_val_pt, const uint8_t* k_scale_pt,
                               const uint8_t* v_val_tb, const uint8_t* v_scale_tb, const uint8_t* v_val_pt,
                               const uint8_t* v_scale_pt, void* o, float* lse, void* ws, size_t ws_bytes,
                               void* stream) {
  int rc = validate_problem(P);
  if (rc != FAPK_OK) return rc;
  if (P->prec != FAPK_MXFP8 || P->d != 128) return FAPK_ERR_UNSUPPORTED;
  if (P->T == 0) return FAPK_OK;
  if (!k_val_tb || !k_scale_tb || !k_val_pt || !k_scale_pt || !aligned16(k_val_tb) || !aligned16(k_val_pt) ||
      (reinterpret_cast<uintptr_t>(k_scale_tb) & 3u) || (reinterpret_cast<uintptr_t>(k_scale_pt) & 3u))
    return FAPK_ERR_INVALID_ARG;
  FwdMxArgs a;
  a.k_vtb = k_val_tb; a.k_stb = k_scale_tb; a.k_vpt = k_val_pt; a.k_spt = k_scale_pt;
  return fwd_quantized_kv(P, q, a, v_val_tb, v_scale_tb, v_val_pt, v_scale_pt, o, lse, ws, ws_bytes, stream);
}

int fapk_attn_fwd_quantized_kv_nvfp4(const fapk_problem_t* P, const void* q, const uint8_t* k_codes,
                                     const uint8_t* k_scales, const uint8_t* v_val_tb, const uint8_t* v_scale_tb,
                                     const uint8_t* v_val_pt, const uint8_t* v_scale_pt, void* o, float* lse,
                                     void* ws, size_t ws_bytes, void* stream) {
  int rc = validate_problem(P);
  if (rc != FAPK_OK) return rc;
  if (P->prec != FAPK_NVFP4_MIXED || P->d != 128) return FAPK_ERR_UNSUPPORTED;
  if (P->T == 0) return FAPK_OK;
  if (!k_codes || !k_scales || !aligned16(k_codes) || (reinterpret_cast<uintptr_t>(k_scales) & 7u))
    return FAPK_ERR_INVALID_ARG;
  FwdMxArgs a;
  a.nv = true;
  a.k_nvv = k_codes;
  a.k_nvs = k_scales;
  a.nv_g_q = nv_scale_of(P->nv_scale_q);
  a.nv_g_k = nv_scale_of(P->nv_scale_k);
  a.k_vtb = a.k_stb = a.k_vpt = a.k_spt = nullptr;  // not read on the mixed path
  return fwd_quantized_kv(P, q, a, v_val_tb, v_scale_tb, v_val_pt, v_scale_pt, o, lse, ws, ws_bytes, stream);
}

int fapk_qkv_proj_mxfp8(const fapk_problem_t* P, const void* x, int d_model, const void* w, void* q, void* k,
                        void* v, uint8_t* k_val_tb, uint8_t* k_scale_tb, uint8_t* k_val_pt, uint8_t* k_scale_pt,
                        uint8_t* v_val_tb, uint8_t* v_scale_tb, uint8_t* v_val_pt, uint8_t* v_scale_pt, void* ws,
                        size_t ws_bytes, void* stream) {
  int rc = validate_problem(P);
  if (rc != FAPK_OK) return rc;
  if (P->prec != FAPK_MXFP8 || P->d != 128) return FAPK_ERR_UNSUPPORTED;
  if (P->T > 0 && (!k_val_tb || !k_scale_tb || !k_val_pt || !k_scale_pt || !aligned16(k_val_tb) ||
                   !aligned16(k_val_pt)))
    return FAPK_ERR_INVALID_ARG;
  QkvProjArgs a;
  a.k_vtb = k_val_tb; a.k_stb = k_scale_tb; a.k_vpt = k_val_pt; a.k_spt = k_scale_pt;
  return qkv_proj(P, x, d_model, w, q, k, v, a, v_val_tb, v_scale_tb, v_val_pt, v_scale_pt, ws, ws_bytes, stream);
}

int fapk_qkv_proj_nvfp4(const fapk_problem_t* P, const void* x, int d_model, const void* w, void* q, void* k,
                        void* v, uint8_t* k_codes, uint8_t* k_scales, uint8_t* v_val_tb, uint8_t* v_scale_tb,
                        uint8_t* v_val_pt, uint8_t* v_scale_pt, void* ws, size_t ws_bytes, void* stream) {
  int rc = validate_problem(P);
  if (rc != FAPK_OK) return rc;
  if (P->prec != FAPK_NVFP4_MIXED || P->d != 128) return FAPK_ERR_UNSUPPORTED;
  if (P->T > 0 && (!k_codes || !k_scales || !aligned16(k_codes) || (reinterpret_cast<uintptr_t>(k_scales) & 1u)))
    return FAPK_ERR_INVALID_ARG;
  QkvProjArgs a;
  a.k_vtb = a.k_stb = a.k_vpt = a.k_spt = nullptr;
  a.k_nvv = k_codes;
  a.k_nvs = k_scales;
  a.nv_g_k = nv_scale_of(P->nv_scale_k);
  return qkv_proj(P, x, d_model, w, q, k, v, a, v_val_tb, v_scale_tb, v_val_pt, v_scale_pt, ws, ws_bytes, stream);
}

int fapk_quantize_mxfp8(const void* x_bf16, int T, int H, int d, const int32_t* cu_seqlens_dev,
                        const int32_t* cu_seqlens_host, int n_docs, int forms, int scale_rule,
                        uint8_t* val_tb, uint8_t* scale_tb, uint8_t* val_pt, uint8_t* scale_pt,
                        void* stream) {
  if (T < 0 || H <= 0 || n_docs < 0) return FAPK_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FAPK_ERR_UNSUPPORTED;
  if (scale_rule != FAPK_SCALE_RCEIL && scale_rule != FAPK_SCALE_OCP) return FAPK_ERR_UNSUPPORTED;
  if ((forms & ~(FAPK_FORM_TB | FAPK_FORM_PT)) != 0 || forms == 0) return FAPK_ERR_INVALID_ARG;
  if (T == 0) return FAPK_OK;
  if (H > 65535 || (long long)T / 32 + n_docs > 0x7FFFFFFFLL) return FAPK_ERR_UNSUPPORTED;
  if (!x_bf16 || !cu_seqlens_dev || n_docs < 1 || !aligned16(x_bf16)) return FAPK_ERR_INVALID_ARG;
  if ((forms & FAPK_FORM_TB) && (!val_tb || !scale_tb)) return FAPK_ERR_INVALID_ARG;
  if ((forms & FAPK_FORM_PT) && (!val_pt || !scale_pt)) return FAPK_ERR_INVALID_ARG;
  if ((val_tb && !aligned16(val_tb)) || (val_pt && !aligned16(val_pt))) return FAPK_ERR_INVALID_ARG;
  if (cu_seqlens_host) {
    if (cu_seqlens_host[0] != 0 || cu_seqlens_host[n_docs] != T) return FAPK_ERR_BAD_SEQLENS;
    for (int k = 0; k < n_docs; ++k)
      if (cu_seqlens_host[k + 1] < cu_seqlens_host[k]) return FAPK_ERR_BAD_SEQLENS;
  }
  return cuda_status(launch_quantize_mxfp8(x_bf16, T, H, d, cu_seqlens_dev, n_docs, forms, scale_rule, val_tb,
                                           scale_tb, val_pt, scale_pt, static_cast<cudaStream_t>(stream)));
}

int fapk_quantize_nvfp4(const void* x_bf16, int T, int H, int d, float g, uint8_t* codes, uint8_t* scales,
                        void* stream) {
  if (T < 0 || H <= 0) return FAPK_ERR_INVALID_ARG;
  if (d != 128) return FAPK_ERR_UNSUPPORTED;
  if (g == 0.f || !nv_scale_ok(g)) return FAPK_ERR_INVALID_ARG;
  if (T == 0) return FAPK_OK;
  if (!x_bf16 || !codes || !scales || !aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(codes) & 7u))
    return FAPK_ERR_INVALID_ARG;
  if ((long long)T * H * 8 > 0x7FFFFFFFLL * 256) return FAPK_ERR_UNSUPPORTED;
  return cuda_status(launch_quantize_nvfp4(x_bf16, T, H, g, codes, scales, static_cast<cudaStream_t>(stream)));
}

int fapk_cta_times(const fapk_problem_t* P, int which, int kernel, const void* ws, void* stream,
                   unsigned long long* out_pairs, int max_ctas, int* n_ctas) {
  if (!P || !ws || !n_ctas || (max_ctas > 0 && !out_pairs) || max_ctas < 0) return FAPK_ERR_INVALID_ARG;
  if (which != FAPK_FWD && which != FAPK_BWD) return FAPK_ERR_INVALID_ARG;
  if (kernel < 0 || kernel > (which == FAPK_FWD ? 0 : 1)) return FAPK_ERR_INVALID_ARG;
  const size_t off = (which == FAPK_FWD ? fwd_layout(P).cta_times : bwd_layout(P).cta_times) +
                     sizeof(unsigned long long) * kCtaTimesWords * (size_t)kernel;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FAPK_ERR_CUDA;
  const char* base = static_cast<const char*>(ws) + off;
  unsigned long long count = 0;
  if (cudaMemcpy(&count, base, sizeof(count), cudaMemcpyDeviceToHost) != cudaSuccess) return FAPK_ERR_CUDA;
  if (count > (unsigned long long)kMaxCtaTimes) count = kMaxCtaTimes;
  *n_ctas = (int)count;
  const int n = (int)count < max_ctas ? (int)count : max_ctas;
  if (n > 0 && cudaMemcpy(out_pairs, base + sizeof(unsigned long long), 2 * sizeof(unsigned long long) * (size_t)n,
                          cudaMemcpyDeviceToHost) != cudaSuccess)
    return FAPK_ERR_CUDA;
  return FAPK_OK;
}

int fapk_status(const void* ws, void* stream) {
  if (!ws) return FAPK_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FAPK_ERR_CUDA;
  DeviceStatus s;
  if (cudaMemcpy(&s, ws, sizeof(s), cudaMemcpyDeviceToHost) != cudaSuccess) return FAPK_ERR_CUDA;
  return s.code;
}

const char* fapk_strerror(int status) {
  switch (status) {
    case FAPK_OK: return "ok";
    case FAPK_ERR_INVALID_ARG: return "invalid argument";
    case FAPK_ERR_UNSUPPORTED: return "unsupported problem (head dim, head grouping or mode)";
    case FAPK_ERR_BAD_SEQLENS: return "malformed cu_seqlens or a document longer than max_seqlen";
    case FAPK_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case FAPK_ERR_CUDA: return "CUDA runtime error";
    case FAPK_ERR_DEVICE_TIMEOUT: return "device watchdog timeout in a pipeline wait";
    case FAPK_ERR_RANGE: return "a value reached 65504, the fp16 range of the P/dS operand path";
    case FAPK_ERR_INTERNAL: return "kernel shared-memory layout check failed";
    default: return "unknown status";
  }
}

uint64_t fapk_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int fapk_version(void) { return 100; }

}  // extern "C"
