/*
 * fapk.h -- C ABI of the causal packed-document flash-attention library for
 * NVIDIA B200 (sm_100a).
 *
 * What it computes.  Exact causal self-attention over packed variable-length
 * documents, forward and backward:
 *   S = scale * Q K^T                 ("GPT Kernel Programlama: MatMul, Softmax
 *                                       ve Attention Hesabi", sec. 3)
 *   key j is visible to query i iff j <= i and both lie in the same document
 *                                      (same page, sec. 4; FLAMIA page, sec.
 *                                       "FLAMIA Mimarisi ve Temel Tasarim
 *                                       Ilkeleri": packed layouts, no repacking)
 *   P = softmax over the visible keys (same page, sec. 5), O = P V (sec. 6),
 * computed tile by tile with an online softmax so that S and P never reach
 * global memory ("FlashAttention (HU)", secs. "Tiling es blokkos
 * feldolgozas", "Online Softmax-szamitas", "Muveletek osszevonasa egyetlen
 * CUDA-kernelbe").  LSE_i = ln sum_j exp(S_ij) (natural log, scale included).
 * The backward is the analytic derivative: D_i = dO_i . O_i, dP = dO V^T,
 * dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
 *
 * Two precisions.  FAPK_BF16: bf16 operands, fp32 accumulation.  FAPK_MXFP8:
 * the FLAMIA page's MXFP8 path -- E4M3 values with one E8M0 scale per 32
 * elements along the contraction, token-block scales reused across the
 * forward and backward orientations, document-local scale blocks, and a leak
 * guard that quantises per token any token block that crosses the causal
 * diagonal (FLAMIA page, same section).
 *
 * Layouts (all row-major, contiguous, device memory, 16-byte aligned):
 *   q, o, dout, dq : [T][Hq][d]      k, v, dk, dv : [T][Hkv][d]
 *   lse            : fp32 [Hq][T]    cu_seqlens   : int32 [n_docs + 1]
 * with cu[0] = 0, cu non-decreasing, cu[n_docs] = T; document k holds tokens
 * [cu[k], cu[k+1]); zero-length documents are allowed and produce nothing.
 * Query head h reads KV head h / (Hq / Hkv).  d must be 64 or 128 (both
 * paths; the MXFP8 path keeps its internal code rows 128 wide and for d = 64
 * fills the upper half with zero codes, which change no real block's scale).
 *
 * Ownership and threading.  The caller owns every buffer (inputs, outputs,
 * workspace, ctx).  The library allocates no device memory and keeps no
 * global state apart from cached kernel attributes; calls on different
 * streams with different workspaces may run concurrently.
 *
 * Execution and errors.  Every call is asynchronous on the given stream
 * (a cudaStream_t passed as void*, NULL for the legacy default stream) and
 * none synchronises, except fapk_status.  A return of FAPK_OK means the work
 * was launched.  Argument errors are detected on the host before anything is
 * launched and returned as codes; nothing is thrown across the ABI and nothing
 * calls exit().  Errors found on the device (a watchdog timeout of a pipeline
 * wait, a document longer than max_seqlen) are written into a status word
 * inside the workspace and read back with fapk_status after the stream's work
 * is done.
 */
#ifndef FAPK_H_
#define FAPK_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FAPK_API __attribute__((visibility("default")))
#else
#define FAPK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
  FAPK_OK = 0,
  FAPK_ERR_INVALID_ARG = 1,         /* null pointer, bad size, misaligned buffer */
  FAPK_ERR_UNSUPPORTED = 2,         /* d not in {64,128}, Hq % Hkv != 0, unknown mode */
  FAPK_ERR_BAD_SEQLENS = 3,         /* cu_seqlens not 0..T non-decreasing, or a document
                                       longer than max_seqlen */
  FAPK_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below fapk_workspace_size() */
  FAPK_ERR_CUDA = 5,                /* a CUDA runtime call failed (launch, no device) */
  FAPK_ERR_DEVICE_TIMEOUT = 6,      /* a bounded device-side wait gave up */
  FAPK_ERR_RANGE = 7,               /* an input or a computed gradient operand reached
                                       65504, the fp16 range of the bf16 path's
                                       P/dS operands (see fapk_attn_fwd) */
  FAPK_ERR_INTERNAL = 8             /* a kernel found its dynamic shared memory not
                                       1024-byte aligned and computed nothing */
} fapk_status_t;

/* Operand precision of the attention path.
 *  FAPK_NVFP4_MIXED: the mixed NVFP4/FP8 path (FLAMIA page, sec. "FLAMIA
 *    Mimarisi ve Temel Tasarim Ilkeleri", which names mixed NVFP4/FP8 training
 *    paths beside MXFP8).  The scores S = Q K^T, in the forward and in the
 *    backward's recomputation alike, take Q and K in NVFP4 (E2M1 codes, one
 *    E4M3 scale per 16 channels of one token, the per-tensor decode scales
 *    nv_scale_q and nv_scale_k; see fapk_quantize_nvfp4); every other
 *    product is the MXFP8 path's (P~ V, dO V^T, and the gradient products
 *    with the MXFP8 forms of K, Q and dO).  d = 64 or 128 (the NVFP4 rows keep
 *    128 channels; for d = 64 the upper 64 are zero codes with scale 0). */
typedef enum { FAPK_BF16 = 0, FAPK_MXFP8 = 1, FAPK_NVFP4_MIXED = 2 } fapk_prec_t;

/* Element type of dq, dk, dv. */
typedef enum { FAPK_GRAD_F32 = 0, FAPK_GRAD_BF16 = 1 } fapk_grad_dtype_t;

/* E8M0 scale-exponent rule of the MXFP8 quantiser.
 *  FAPK_SCALE_RCEIL (default): X = ceil(log2(amax / 448)), the smallest
 *    exponent at which the block maximum fits E4M3 without saturating.
 *  FAPK_SCALE_OCP: X = floor(log2(amax)) - 8 (OCP Microscaling v1.0);
 *    block maxima whose mantissa exceeds 1.75 saturate to 448.
 * Both clamp X to [-127, 127]; an all-zero block takes X = -127.  The scale
 * byte is X + 127.  fapk_quantize_mxfp8 takes either rule.  The MXFP8
 * attention path takes RCEIL only (FAPK_ERR_UNSUPPORTED otherwise): under
 * OCP a computed P or dS block whose maximum lies just below a power of two
 * saturates (up to 12.5% error) while one just above does not, so the
 * gradients jump with tiny changes of P (a 1e-6 relative change of P moved
 * dV by 2.8% in a measured case), and OCP is further from exact fp64 than
 * RCEIL on every output. */
typedef enum { FAPK_SCALE_RCEIL = 0, FAPK_SCALE_OCP = 1 } fapk_scale_rule_t;

/* Which pass a workspace is sized for. */
enum { FAPK_FWD = 0, FAPK_BWD = 1 };

/* Forms produced by fapk_quantize_mxfp8 (bit mask). */
enum { FAPK_FORM_TB = 1, FAPK_FORM_PT = 2 };

/* Debug flags (fapk_problem_t.flags). */
enum {
  /* Fault injection for the watchdog test: the forward's load producer drops
   * one K/V tile copy, so the consumer's bounded wait runs out and the call
   * reports FAPK_ERR_DEVICE_TIMEOUT through fapk_status.  No fault, trap or
   * hang is involved. */
  FAPK_FLAG_INJECT_DROP_LOAD = 1 << 0,
  /* Scheduler balance: every CTA of the call's persistent attention kernels
   * records the %globaltimer (ns) when it starts and when it has finished its
   * work units, in the workspace; read them back with fapk_cta_times. */
  FAPK_FLAG_CTA_TIMES = 1 << 1
};

/* One attention problem.  All fields are read during the call only. */
typedef struct {
  int T;                         /* total packed tokens (>= 0) */
  int n_docs;                    /* number of documents (>= 1 when T > 0) */
  int max_seqlen;                /* upper bound of any document length (>= 1 when T > 0) */
  int Hq, Hkv, d;                /* query heads, KV heads (Hq % Hkv == 0), head dim (64|128) */
  float scale;                   /* softmax scale, usually 1/sqrt(d) */
  int prec;                      /* fapk_prec_t */
  int scale_rule;                /* fapk_scale_rule_t (MXFP8 path) */
  const int32_t* cu_seqlens_dev; /* device copy of cu_seqlens (required) */
  const int32_t* cu_seqlens_host;/* host copy; when non-NULL it is validated on the host */
  int grad_dtype;                /* fapk_grad_dtype_t of dq, dk, dv */
  int flags;                     /* debug flags, 0 in normal use */
  int timeout_ms;                /* device watchdog per wait; <= 0 selects 2000 ms */
  void* const* timing_events;    /* optional profiling hook: cudaEvent_t handles that a call
                                    records on its stream before each of its kernel launches
                                    and after the last one (entries beyond n_timing_events or
                                    NULL are skipped).  fapk_attn_fwd: [0] schedule, [1] fp16
                                    copy of V (FAPK_MXFP8: MX quantisation of K and V),
                                    [2] forward kernel, [3] end.  fapk_attn_bwd, FAPK_BF16:
                                    [0] key-tile schedule, [1] query-tile schedule, [2] fp16
                                    copy of K, [3] D and fp16 dO/Q, [4] dK/dV kernel, [5] dQ
                                    kernel, [6] end; FAPK_MXFP8: [0] key-tile schedule,
                                    [1] query-tile schedule, [2] D and MX quantisation of dO,
                                    [3] dK/dV kernel, [4] dQ kernel, [5] end. */
  int n_timing_events;
  float nv_scale_q, nv_scale_k;  /* FAPK_NVFP4_MIXED: per-tensor fp32 decode scales g of
                                    Q and K (0 selects 1; else within [2^-100, 2^100],
                                    FAPK_ERR_INVALID_ARG otherwise).  They are the
                                    caller's, e.g. from earlier steps' maxima: a scale
                                    taken from this batch's tensor-wide maximum would
                                    let later tokens set the codes of earlier ones. */
} fapk_problem_t;

/* Bytes of workspace the forward (which = FAPK_FWD) or backward
 * (which = FAPK_BWD) needs for this problem; 0 if the problem is invalid.
 * The workspace is scratch owned by the caller: device memory, 256-byte
 * aligned, contents need not be initialised, not shared by concurrent calls. */
FAPK_API size_t fapk_workspace_size(const fapk_problem_t* prob, int which);

/* Bytes of the saved-state buffer `ctx` that the forward fills and the
 * backward reads.  It holds the bf16 rounding residual of O (O_fp32 minus its
 * bf16 rounding, [T][Hq][d] bf16), so that the backward's D_i = dO_i . O_i
 * sees O to about 16 significant bits; the bf16 path adds an fp16 copy of V,
 * the MXFP8 path the MX forms (codes and scales, token-block and per-token) of
 * Q, K and V, reused across orientations (FLAMIA page: "token-block
 * scaling"); the mixed NVFP4/FP8 path adds the NVFP4 forms of Q and K. */
FAPK_API size_t fapk_ctx_size(const fapk_problem_t* prob);

/* Forward.  Reads q, k, v (bf16); writes o (bf16) and lse (fp32, natural
 * log).  ctx (required): device buffer of fapk_ctx_size() bytes, 16-byte
 * aligned, filled for the backward.  ws: workspace of at least
 * fapk_workspace_size(prob, FAPK_FWD) bytes.
 * FAPK_BF16 numerics: S = Q K^T on bf16 operands with fp32 accumulation; the
 * probabilities P (computed in fp32) multiply V as fp16 operands, which keep
 * 11 significant bits where bf16 keeps 8 (a bf16 value converts to fp16
 * exactly when its magnitude is below 65504).  Inputs reaching 65504 in
 * magnitude are reported as FAPK_ERR_RANGE by fapk_status. */
FAPK_API int fapk_attn_fwd(const fapk_problem_t* prob, const void* q, const void* k, const void* v,
                  void* o, float* lse, void* ctx, void* ws, size_t ws_bytes, void* stream);

/* Backward.  Reads q, k, v, o, lse, dout (bf16 except lse) and the ctx
 * written by the matching forward (required); every MMA of the FAPK_BF16
 * backward runs on fp16 operands (P and dS with 11 significant bits), and a
 * |dS| reaching 65504 is reported as FAPK_ERR_RANGE; writes dq [T][Hq][d] and
 * dk, dv [T][Hkv][d] in grad_dtype.  dk and dv are summed over the query
 * heads that share a KV head.  ws: at least fapk_workspace_size(prob,
 * FAPK_BWD) bytes. */
FAPK_API int fapk_attn_bwd(const fapk_problem_t* prob, const void* q, const void* k, const void* v,
                  const void* o, const float* lse, const void* dout, const void* ctx,
                  void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, void* stream);

/* MXFP8 quantisation of a bf16 tensor x [T][H][d] (FLAMIA page: MXFP8,
 * token-block scaling, document-local scaling).  E4M3 codes (round to nearest
 * even, saturating to +-448, a zero result is always code 0x00) and E8M0
 * scale bytes.
 *   forms & FAPK_FORM_TB: token-block form.  One scale per 32 tokens x 32
 *     channels of one head; token blocks are document-local: block m of
 *     document k covers tokens [s_k + 32m, min(s_k + 32m + 32, e_k)).
 *     val_tb [T][H][d] codes; scale_tb [T/32 + n_docs][H][d/32] scale bytes,
 *     block m of document k in slot floor(s_k/32) + k + m (slots holding no
 *     block are not written).
 *   forms & FAPK_FORM_PT: per-token form.  One scale per token x 32 channels.
 *     val_pt [T][H][d]; scale_pt [T][H][d/32].
 * Pointers of a form not requested may be NULL.  x must be 16-byte aligned;
 * d is 64 or 128. */
FAPK_API int fapk_quantize_mxfp8(const void* x_bf16, int T, int H, int d, const int32_t* cu_seqlens_dev,
                        const int32_t* cu_seqlens_host, int n_docs, int forms, int scale_rule,
                        uint8_t* val_tb, uint8_t* scale_tb, uint8_t* val_pt, uint8_t* scale_pt,
                        void* stream);

/* NVFP4 quantisation of a bf16 tensor x [T][H][d] (d = 128), the operand
 * form of the mixed NVFP4/FP8 path's scores.  NVFP4 is NVIDIA's published
 * format (the FLAMIA page only names it): E2M1 codes, one unsigned E4M3
 * scale per 16 consecutive channels of one token, and the per-tensor fp32
 * decode scale g, x ~ code * scale * g.  A block with largest magnitude a is
 * quantised in fp32 arithmetic, each step rounded to nearest even:
 *   s = E4M3(a / (6 g))     (saturating at 448; 0 for an all-zero block),
 *   r = 1 / (decode(s) g)   (0 when that product is 0),
 *   code_i = E2M1(x_i r)    (saturating at +-6; a zero result is code 0).
 * codes [T][H][d/2] (channel 2i in the low nibble of byte i), 8-byte
 * aligned; scales [T][H][d/16].  g must be finite and within [2^-100,
 * 2^100] (FAPK_ERR_INVALID_ARG); x 16-byte aligned.  The attention path's
 * own NVFP4 operands are computed with the same arithmetic (K by its
 * prepass, Q on load by the forward kernel). */
FAPK_API int fapk_quantize_nvfp4(const void* x_bf16, int T, int H, int d, float g, uint8_t* codes,
                                 uint8_t* scales, void* stream);

/* MXFP8 forward over already-quantised K and V ("Flash Attention" glossary
 * page on local inference engines, secs. "Tanim" and the KV-cache table: a
 * quantised KV cache, read directly by the fused attention kernel, holds the
 * keys and values in half the bytes of f16).  Q is bf16 and quantised on load
 * as in fapk_attn_fwd; K and V arrive in both MX forms exactly as
 * fapk_quantize_mxfp8 writes them (forms = FAPK_FORM_TB | FAPK_FORM_PT, for
 * example once into a cache and then reused by many calls), so the call
 * launches no quantisation of its own.  Inference only: no ctx, no backward.
 *  - prob->prec must be FAPK_MXFP8, prob->d 128 (FAPK_ERR_UNSUPPORTED
 *    otherwise); the forms must have been made with prob's cu_seqlens and
 *    scale rule.
 *  - k_val_tb, k_val_pt, v_val_tb, v_val_pt: codes [T][Hkv][128], 16-byte
 *    aligned; k_scale_tb, v_scale_tb: [T/32 + n_docs][Hkv][4];
 *    k_scale_pt, v_scale_pt: [T][Hkv][4]; scales 4-byte aligned.
 *  - q, o, lse, ws and errors as in fapk_attn_fwd.  With the forms of
 *    fapk_quantize_mxfp8, O and LSE are bit-identical to fapk_attn_fwd's in
 *    the MXFP8 path. */
FAPK_API int fapk_attn_fwd_quantized_kv(const fapk_problem_t* prob, const void* q, const uint8_t* k_val_tb,
                                        const uint8_t* k_scale_tb, const uint8_t* k_val_pt,
                                        const uint8_t* k_scale_pt, const uint8_t* v_val_tb,
                                        const uint8_t* v_scale_tb, const uint8_t* v_val_pt,
                                        const uint8_t* v_scale_pt, void* o, float* lse, void* ws,
                                        size_t ws_bytes, void* stream);

/* Fused QKV projection with MXFP8 quantisation of K and V in its epilogue
 * ("GPT Kernel Programlama: MatMul, Softmax ve Attention Hesabi", sec. 2: the
 * three projections as one fused QKV projection; FLAMIA page, sec. "FLAMIA
 * Mimarisi ve Temel Tasarim Ilkeleri": fused quantisation, document-local
 * scales over packed layouts).  One tensor-core GEMM [Q | K | V] = X W^T over
 * the packed tokens:
 *   x: [T][d_model] bf16 (d_model a multiple of 8);
 *   w: [(Hq + 2 Hkv) d][d_model] bf16, the rows of the Q heads, then the K
 *      heads, then the V heads (the usual out x in layout of a linear layer);
 *   q: [T][Hq][d], k, v: [T][Hkv][d] bf16, the fp32 products rounded to
 *      nearest even;
 *   K's and V's token-block and per-token MX forms, quantised from those bf16
 *   values with prob's cu_seqlens and scale rule, in the layout of
 *   fapk_quantize_mxfp8 (codes [T][Hkv][128], 16-byte aligned; scales
 *   [T/32 + n_docs][Hkv][4] and [T][Hkv][4]), ready for
 *   fapk_attn_fwd_quantized_kv, which then launches no quantisation.
 * prob->prec must be FAPK_MXFP8 and prob->d 128 (FAPK_ERR_UNSUPPORTED
 * otherwise).  ws: at least fapk_workspace_size(prob, FAPK_FWD) bytes (the
 * same work order as the MXFP8 forward).  Asynchronous like the other calls;
 * the device status word is read with fapk_status(ws). */
FAPK_API int fapk_qkv_proj_mxfp8(const fapk_problem_t* prob, const void* x, int d_model, const void* w,
                                 void* q, void* k, void* v, uint8_t* k_val_tb, uint8_t* k_scale_tb,
                                 uint8_t* k_val_pt, uint8_t* k_scale_pt, uint8_t* v_val_tb,
                                 uint8_t* v_scale_tb, uint8_t* v_val_pt, uint8_t* v_scale_pt, void* ws,
                                 size_t ws_bytes, void* stream);

/* The mixed NVFP4/FP8 path's counterparts of the two calls above (prob->prec
 * = FAPK_NVFP4_MIXED, d = 128; otherwise FAPK_ERR_UNSUPPORTED).
 *  fapk_qkv_proj_nvfp4: the same projection, with K's NVFP4 form in place of
 *    its MX forms: k_codes [T][Hkv][64] (16-byte aligned) and k_scales
 *    [T][Hkv][8] (2-byte aligned), quantised from the bf16 K with decode
 *    scale prob->nv_scale_k exactly as fapk_quantize_nvfp4 would; V's MX
 *    forms as above.
 *  fapk_attn_fwd_quantized_kv_nvfp4: the mixed path's forward over K in
 *    NVFP4 (k_codes, k_scales as fapk_quantize_nvfp4 or the projection write
 *    them; 16- and 8-byte aligned) and V in both MX forms; Q is quantised on
 *    load as in fapk_attn_fwd.  No quantisation launch and no saved state;
 *    the output is bit-identical to fapk_attn_fwd's on the same inputs.
 * Ownership, workspace, stream and errors as for the MXFP8 calls. */
FAPK_API int fapk_qkv_proj_nvfp4(const fapk_problem_t* prob, const void* x, int d_model, const void* w,
                                 void* q, void* k, void* v, uint8_t* k_codes, uint8_t* k_scales,
                                 uint8_t* v_val_tb, uint8_t* v_scale_tb, uint8_t* v_val_pt,
                                 uint8_t* v_scale_pt, void* ws, size_t ws_bytes, void* stream);
FAPK_API int fapk_attn_fwd_quantized_kv_nvfp4(const fapk_problem_t* prob, const void* q,
                                              const uint8_t* k_codes, const uint8_t* k_scales,
                                              const uint8_t* v_val_tb, const uint8_t* v_scale_tb,
                                              const uint8_t* v_val_pt, const uint8_t* v_scale_pt, void* o,
                                              float* lse, void* ws, size_t ws_bytes, void* stream);

/* Forward that allocates nothing.  The pages have no counterpart: this entry
 * point exists for callers that cannot obtain device memory where they run the
 * forward -- a plugin handed its buffers by a host framework that must not
 * allocate on its own, or a runtime that reserves all device memory at
 * start-up.  Same arguments and results as fapk_attn_fwd minus the workspace:
 * inputs, outputs and ctx are still the caller's, and the forward's scratch
 * (status word and work list) is a 1 MiB array of device memory inside the
 * library, which every GPU that loads the library holds until the process
 * exits.
 *  - A problem whose forward workspace (fapk_workspace_size(prob, FAPK_FWD))
 *    exceeds 1 MiB is rejected with FAPK_ERR_WORKSPACE_TOO_SMALL.  That size
 *    is about 17 KiB, plus 12 bytes per ceil(max_seqlen / 128) and 8 bytes
 *    per document: at most about 128 800 documents fit.
 *  - The first call on a device looks up the array's device address with that
 *    device current; under CUDA's lazy module loading (the default) this is
 *    also when the array's 1 MiB is taken on that device.  Make that first
 *    call before any stream capture and before reserving the rest of the
 *    device's memory.
 *  - It makes CUDA runtime calls, so it must not be called from inside a
 *    stream callback (cudaLaunchHostFunc / cudaStreamAddCallback).
 *  - All calls share the array and it keeps the last call's contents; each
 *    call clears the status word and counters it uses when it starts.  Calls
 *    whose GPU work overlaps (different streams or host threads) race on it.
 *  - The device status word is read with fapk_noalloc_status. */
FAPK_API int fapk_attn_fwd_noalloc(const fapk_problem_t* prob, const void* q, const void* k,
                                   const void* v, void* o, float* lse, void* ctx, void* stream);

/* Device status word of the last fapk_attn_fwd_noalloc call on the current
 * device: synchronises `stream`, then returns FAPK_OK, FAPK_ERR_DEVICE_TIMEOUT
 * or FAPK_ERR_BAD_SEQLENS as fapk_status does for a workspace, or
 * FAPK_ERR_CUDA if the stream reported an error.  Allocates nothing. */
FAPK_API int fapk_noalloc_status(void* stream);

/* Scheduler balance (the pages have no counterpart): after a call made with
 * FAPK_FLAG_CTA_TIMES on workspace `ws` and problem `prob`, synchronises
 * `stream` and copies, for the call's persistent kernel number `kernel`
 * (forward, which = FAPK_FWD: 0 = the attention kernel; backward, which =
 * FAPK_BWD: 0 = dK/dV, 1 = dQ), one (start, end) pair of %globaltimer values
 * in ns per CTA into out_pairs[2 * i], out_pairs[2 * i + 1] for the first
 * min(CTAs, max_ctas) CTAs; *n_ctas receives the kernel's CTA count.
 * Host-owned output; FAPK_ERR_INVALID_ARG for a bad kernel number or null
 * pointer, FAPK_ERR_CUDA if the copy fails. */
FAPK_API int fapk_cta_times(const fapk_problem_t* prob, int which, int kernel, const void* ws, void* stream,
                            unsigned long long* out_pairs, int max_ctas, int* n_ctas);

/* Synchronises `stream`, then returns the device status word of the last call
 * that used workspace `ws` (FAPK_OK, FAPK_ERR_DEVICE_TIMEOUT, or
 * FAPK_ERR_BAD_SEQLENS), or FAPK_ERR_CUDA if the stream reported an error. */
FAPK_API int fapk_status(const void* ws, void* stream);

/* Static text for a status code. */
FAPK_API const char* fapk_strerror(int status);

/* Number of kernels this library has launched in this process (all threads). */
FAPK_API uint64_t fapk_launch_count(void);

/* Library version, major * 10000 + minor * 100 + patch. */
FAPK_API int fapk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FAPK_H_ */
