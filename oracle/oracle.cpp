/*
 * fapk oracle -- a plain, slow fp64 CPU reference for causal attention over
 * packed variable-length documents, forward and backward, plus an emulation of
 * the MXFP8 quantisation rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path; the only thing the two sides
 * have in common is the seeded input generator, which holds no arithmetic of
 * the method.
 *
 * Sources, cited by page title and section:
 *  [GPT]    "GPT Kernel Programlama: MatMul, Softmax ve Attention Hesabi"
 *           sec. 3 (S[i,j] = sum_r Q[i,r] K[j,r] / sqrt(d)), sec. 4 (causal
 *           mask: j > i is excluded), sec. 5 (stable softmax: subtract the
 *           row maximum, exponentiate, divide by the sum), sec. 6
 *           (O[i,r] = sum_j P[i,j] V[j,r]), sec. 7 (fused/tiled attention
 *           gives the same result, no approximation).
 *  [FLAMIA] "FLAMIA: Blackwell Uzerinde Hizli ve Nedensel Olarak Guvenli
 *           Egitim Icin Flash Mikro-Olceklemeli Dikkat Mekanizmasi",
 *           sec. "FLAMIA Mimarisi ve Temel Tasarim Ilkeleri": MXFP8 path,
 *           token-block scaling reused across orientations, leak guards
 *           (no information from future tokens through shared scales),
 *           forward/backward consistency, document-local scaling over packed
 *           layouts without repacking.
 *  [FA-HU]  "FlashAttention (HU)", sec. "Online Softmax-szamitas": tiling with
 *           a running max/sum reaches exactly the softmax result.  The oracle
 *           does NOT tile: it materialises one score row per query.
 *
 * Readings where the pages are silent (the choices this oracle makes):
 *  - packed documents: token i of document k=[s_k,e_k) sees keys j with
 *    s_k <= j <= i only; cu_seqlens gives s_k = cu[k], e_k = cu[k+1].
 *  - GQA: query head h reads KV head h / (Hq/Hkv).
 *  - LSE_i = m_i + ln(l_i): natural log, softmax scale included.
 *  - backward = analytic derivative (the pages give no formulas):
 *    D_i = dO_i . O_i, dP_ij = dO_i . V_j, dS_ij = P_ij (dP_ij - D_i),
 *    dQ_i = s sum_j dS_ij K_j, dK_j = s sum_i dS_ij Q_i, dV_j = sum_i P_ij dO_i.
 *  - MXFP8: E4M3 element codes, E8M0 shared scale per 32 elements, element
 *    code = RNE(x * 2^-X) saturated to +-448, scale byte X + 127.  Scale
 *    exponent (block_exponent below), clamped to [-127, 127], X = -127 for an
 *    all-zero block:
 *      RULE_RCEIL (the default): X = ceil(log2(amax / 448)), the smallest
 *        exponent at which the block maximum does not saturate;
 *      RULE_OCP (flag MX_RULE_OCP): X = floor(log2 amax) - 8, the OCP
 *        Microscaling v1.0 rule, under which block maxima whose significand
 *        exceeds 1.75 saturate to 448.
 *    (Block size and formats from the benchmark spec.)
 *  - mixed NVFP4/FP8 path ([FLAMIA] names "mixed NVFP4/FP8 training paths"
 *    without giving the split): the scores S = Q K^T, in the forward and in
 *    the backward's recomputation alike (fwd/bwd consistency), take Q and K
 *    in NVFP4; every other product is the MXFP8 path's.  NVFP4 is NVIDIA's
 *    published format (the pages only name it): E2M1 element codes, one
 *    unsigned E4M3 scale per 16 consecutive channels of one token, and one
 *    fp32 decode scale g per tensor, x ~ code * scale * g.  Quantisation of a
 *    block with largest magnitude a, in fp32 arithmetic (each step rounded to
 *    nearest even):  s = E4M3(a / (6 g)) (saturating at 448),
 *    r = 1 / (decode(s) g) (0 when that is 0), code_i = E2M1(x_i r)
 *    (saturating at 6; a zero result is code 0).  g is the caller's (a
 *    tensor-wide amax of this batch would let later tokens set the scale of
 *    earlier ones); the blocks lie along channels inside one token, so no
 *    leak guard is needed for them.
 *  - token blocks are document-local: block m of document k covers tokens
 *    [s_k + 32m, min(s_k + 32m + 32, e_k)); its scale lives in slot
 *    floor(s_k/32) + k + m of a [T/32 + n_docs] slot array.
 *  - leak guard (rule L): a shared scale may not pool a token that the output
 *    it influences must not see.  Key-side operands (K in Q K^T and in
 *    dQ = dS K, V in P V and in dP = dO V^T) are taken in token-block form
 *    (32 tokens x 32 channels share one scale) for key blocks before the
 *    query's block and in per-token form (one scale per token x 32 channels)
 *    on the diagonal block; Q in Q K^T and dO in dO V^T are always per-token.
 *    Query-side operands of the query contraction (Q in dK = dS^T Q, dO in
 *    dV = P^T dO) are in token-block form in every query block: every query
 *    with a non-zero term there is causally after the key.  Computed P and dS
 *    are quantised per 32-block along their contraction (P, dS per (query row,
 *    key block); P^T, dS^T per (key row, query block)), from the normalised
 *    fp64 P.
 *
 * Parity pins (tests/test_oracle_*.py): Q=0 closed forms, one-token
 * documents, constant V, rows summing to one, torch fp64 SDPA on one
 * document, packing and permutation invariance, central finite differences
 * of the backward, brute force of the quantiser over every finite bf16 value,
 * the E4M3 round trip, worked quantiser values, the MXFP8 emulation's
 * exact limit, its cosine to the exact path and the leak properties; the
 * forward P~ of a hand-derived row and its independence of the integer
 * reference; the blocks of dS~, P~T and dS~T read out element by element
 * (document-local, along the contraction); the operand forms of dP (dO per
 * token) and of dK, dV (Q, dO in token-block form) in hand-derived cases.
 */
#include <algorithm>
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

struct Problem {
  int T, nd, Hq, Hkv, d;
  const int32_t* cu;
  double scale;
  int G() const { return Hq / Hkv; }
};

inline size_t idx3(int t, int h, int r, int H, int d) {
  return ((size_t)t * H + h) * d + r;
}

/* ------------------------------------------------------------------------ */
/* Exact attention: one materialised score row per query [GPT] sec. 3-6.     */
/* ------------------------------------------------------------------------ */

/* Scores of query row i (global token index) of head h against the keys
 * s..i of its own document, then the stable softmax of [GPT] sec. 5.
 * Kt is K of this (document, kv head) transposed to [d][L] so that each
 * score S_ij = scale * sum_{r=0..d-1} Q_ir K_jr is still summed over r in
 * order 0..d-1 (the loop over j is the vectorised one).
 * Outputs: p[0..n) = normalised P_ij for j = s..i, m = row max, l = row sum of
 * exp(S - m).  Returns n = i - s + 1. */
int score_row(const double* qi, const std::vector<double>& Kt, int L, int d, int li,
              double scale, std::vector<double>& srow, std::vector<double>& p, double& m,
              double& l) {
  const int n = li + 1;
  srow.assign(n, 0.0);
  for (int r = 0; r < d; ++r) {
    const double qr = qi[r];
    const double* kr = &Kt[(size_t)r * L];
    for (int j = 0; j < n; ++j) srow[j] += qr * kr[j];
  }
  m = -INFINITY;
  for (int j = 0; j < n; ++j) {
    srow[j] *= scale;
    m = std::max(m, srow[j]);
  }
  p.resize(n);
  l = 0.0;
  for (int j = 0; j < n; ++j) {
    p[j] = std::exp(srow[j] - m);
    l += p[j];
  }
  for (int j = 0; j < n; ++j) p[j] /= l;
  return n;
}

/* Transposed copy of one (document, head) slice of a [T][H][d] tensor. */
void slice_t(const double* x, int s, int L, int h, int H, int d, std::vector<double>& out) {
  out.assign((size_t)d * L, 0.0);
  for (int j = 0; j < L; ++j)
    for (int r = 0; r < d; ++r) out[(size_t)r * L + j] = x[idx3(s + j, h, r, H, d)];
}

/* Row-major copy of one (document, head) slice: [L][d]. */
void slice_n(const double* x, int s, int L, int h, int H, int d, std::vector<double>& out) {
  out.resize((size_t)L * d);
  for (int j = 0; j < L; ++j)
    for (int r = 0; r < d; ++r) out[(size_t)j * d + r] = x[idx3(s + j, h, r, H, d)];
}

struct Task {
  int doc, h;
  double cost;
};

std::vector<Task> head_doc_tasks(const Problem& P, int nheads) {
  std::vector<Task> t;
  for (int k = 0; k < P.nd; ++k) {
    const double L = P.cu[k + 1] - P.cu[k];
    if (L <= 0) continue;
    for (int h = 0; h < nheads; ++h) t.push_back({k, h, L * L});
  }
  std::stable_sort(t.begin(), t.end(), [](const Task& a, const Task& b) { return a.cost > b.cost; });
  return t;
}

/* Exact forward of one (document, query head): O rows and LSE. */
void fwd_doc_head(const Problem& P, int k, int h, const double* q, const double* kk,
                  const double* v, double* o, double* lse) {
  const int s = P.cu[k], L = P.cu[k + 1] - P.cu[k], d = P.d, g = h / P.G();
  std::vector<double> Kt, Vn, srow, p;
  slice_t(kk, s, L, g, P.Hkv, d, Kt);
  slice_n(v, s, L, g, P.Hkv, d, Vn);
  std::vector<double> orow(d);
  for (int li = 0; li < L; ++li) {
    const int i = s + li;
    double m, l;
    const int n = score_row(&q[idx3(i, h, 0, P.Hq, d)], Kt, L, d, li, P.scale, srow, p, m, l);
    std::fill(orow.begin(), orow.end(), 0.0);
    for (int j = 0; j < n; ++j) {
      const double pj = p[j];
      const double* vj = &Vn[(size_t)j * d];
      for (int r = 0; r < d; ++r) orow[r] += pj * vj[r];
    }
    for (int r = 0; r < d; ++r) o[idx3(i, h, r, P.Hq, d)] = orow[r];
    lse[(size_t)h * P.T + i] = m + std::log(l);
  }
}

/* ------------------------------------------------------------------------ */
/* MXFP8 emulation: E4M3 codes with an E8M0 scale per 32-element block.     */
/* ------------------------------------------------------------------------ */

/* floor(log2 a) for a > 0, read from the binary exponent (frexp), never from a
 * floating-point logarithm. */
inline int floor_log2(double a) {
  int e;
  std::frexp(a, &e);  // a = f * 2^e, f in [0.5, 1)
  return e - 1;
}

/* Scale-exponent rules.
 *  RULE_RCEIL (default): the smallest X with amax * 2^-X <= 448, i.e.
 *    X = ceil(log2(amax / 448)); the block maximum never saturates.
 *  RULE_OCP: X = floor(log2 amax) - 8 (the OCP Microscaling v1.0 rule for
 *    E4M3); a block maximum whose mantissa exceeds 1.75 saturates to 448.
 * Both clamp X to [-127, 127]; an all-zero block takes X = -127. */
enum { RULE_RCEIL = 0, RULE_OCP = 1 };

/* Shared scale exponent X of a block whose largest magnitude is amax. */
inline int block_exponent(double amax, int rule) {
  if (amax == 0.0) return -127;
  const int e = floor_log2(amax);
  int X = e - 8;
  if (rule == RULE_RCEIL && amax > 1.75 * std::ldexp(1.0, e)) X += 1;
  return std::min(127, std::max(-127, X));
}

/* Round half to even of a non-negative value (exact in fp64 here). */
inline double rne(double n) {
  const double f = std::floor(n);
  const double frac = n - f;
  if (frac > 0.5) return f + 1.0;
  if (frac < 0.5) return f;
  return (std::fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* E4M3 code of y (already divided by the block scale): round to nearest,
 * ties to even, saturate to +-448; bias 7, subnormals down to 2^-9, no
 * infinity; a zero result is always code 0x00. */
uint8_t e4m3_encode(double y) {
  const uint8_t sign = (y < 0.0) ? 0x80 : 0x00;
  double a = std::fabs(y);
  if (a >= 448.0) return sign | 0x7E;  // 1.75 * 2^8
  if (a == 0.0) return 0x00;
  int e = floor_log2(a);
  if (e < -6) e = -6;  // subnormal range shares the quantum 2^-9
  const double quantum = std::ldexp(1.0, e - 3);
  const double qv = rne(a / quantum) * quantum;
  if (qv == 0.0) return 0x00;
  const int e2 = floor_log2(qv);
  uint8_t ef, mf;
  if (e2 < -6) {
    ef = 0;
    mf = (uint8_t)(qv / std::ldexp(1.0, -9));
  } else {
    ef = (uint8_t)(e2 + 7);
    mf = (uint8_t)(qv / std::ldexp(1.0, e2) * 8.0 - 8.0);
  }
  return sign | (uint8_t)(ef << 3) | mf;
}

double e4m3_decode(uint8_t c) {
  const int ef = (c >> 3) & 15, mf = c & 7;
  double v;
  if ((c & 0x7F) == 0x7F) return NAN;
  if (ef == 0)
    v = mf * std::ldexp(1.0, -9);
  else
    v = (1.0 + mf / 8.0) * std::ldexp(1.0, ef - 7);
  return (c & 0x80) ? -v : v;
}

/* Quantise the n values x[0], x[stride], ... as one block; writes codes and
 * the dequantised values (decode(code) * 2^X); returns the scale byte. */
uint8_t quant_block(const double* x, int n, size_t stride, uint8_t* codes, size_t cstride,
                    double* deq, size_t dstride, int rule) {
  double amax = 0.0;
  for (int t = 0; t < n; ++t) amax = std::max(amax, std::fabs(x[t * stride]));
  const int X = block_exponent(amax, rule);
  for (int t = 0; t < n; ++t) {
    const uint8_t c = e4m3_encode(std::ldexp(x[t * stride], -X));
    if (codes) codes[t * cstride] = c;
    if (deq) deq[t * dstride] = std::ldexp(e4m3_decode(c), X);
  }
  return (uint8_t)(X + 127);
}

/* Token-block (tb) and per-token (pt) dequantised forms of one (document,
 * head) slice, row-major [L][d] in doc-local token order.  With `exact` (an
 * accuracy-study switch) both forms are the unquantised values. */
void mx_forms(const double* x, int s, int L, int h, int H, int d, int rule,
              std::vector<double>& tb, std::vector<double>& pt, bool exact = false) {
  std::vector<double> xs;
  slice_n(x, s, L, h, H, d, xs);
  if (exact) {
    tb = xs;
    pt = xs;
    return;
  }
  tb.assign((size_t)L * d, 0.0);
  pt.assign((size_t)L * d, 0.0);
  for (int j = 0; j < L; ++j)
    for (int c0 = 0; c0 < d; c0 += 32)
      quant_block(&xs[(size_t)j * d + c0], 32, 1, nullptr, 0, &pt[(size_t)j * d + c0], 1, rule);
  for (int b0 = 0; b0 < L; b0 += 32) {
    const int nb = std::min(32, L - b0);
    for (int c0 = 0; c0 < d; c0 += 32) {
      // one scale for the nb x 32 tile: the amax is taken over all of it
      double amax = 0.0;
      for (int j = b0; j < b0 + nb; ++j)
        for (int c = c0; c < c0 + 32; ++c) amax = std::max(amax, std::fabs(xs[(size_t)j * d + c]));
      const int X = block_exponent(amax, rule);
      for (int j = b0; j < b0 + nb; ++j)
        for (int c = c0; c < c0 + 32; ++c) {
          const uint8_t code = e4m3_encode(std::ldexp(xs[(size_t)j * d + c], -X));
          tb[(size_t)j * d + c] = std::ldexp(e4m3_decode(code), X);
        }
    }
  }
}

/* ---- NVFP4 (mixed path) ------------------------------------------------- */

/* E2M1 code of y: round to nearest, ties to the even code, saturate to +-6;
 * 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit: magnitudes
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7.  A zero result is code 0. */
uint8_t e2m1_encode(double y) {
  const double a = std::fabs(y);
  double qv;
  if (a >= 6.0) {
    qv = 6.0;
  } else {
    const int e = a < 1.0 ? 0 : floor_log2(a);     // below 1: the subnormal quantum 0.5
    const double quantum = std::ldexp(1.0, e - 1);  // one mantissa bit
    qv = std::min(6.0, rne(a / quantum) * quantum);
  }
  if (qv == 0.0) return 0;
  uint8_t mag;
  if (qv < 1.0)
    mag = 1;  // 0.5, subnormal
  else {
    const int e2 = floor_log2(qv);
    mag = (uint8_t)(((e2 + 1) << 1) | (qv > std::ldexp(1.0, e2) ? 1 : 0));
  }
  return (uint8_t)((y < 0.0 ? 8 : 0) | mag);
}

double e2m1_decode(uint8_t c) {
  const int mag = c & 7, e = mag >> 1, m = mag & 1;
  const double v = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return (c & 8) ? -v : v;
}

/* One NVFP4 block of n (16) values x[0..n) (bf16 values, exact in fp32) with
 * the tensor's decode scale g: codes (E2M1, one per value), dequantised
 * values code * decode(s) * g (fp64), returns the E4M3 scale byte s.  The
 * arithmetic is fp32, step by step as the format's quantisation states it. */
uint8_t nv_quant_block(const double* x, int n, float g, uint8_t* codes, double* deq) {
  float a = 0.f;
  for (int i = 0; i < n; ++i) a = std::max(a, std::fabs((float)x[i]));
  const float six_g = 6.0f * g;
  const float t = a / six_g;
  const uint8_t sbyte = e4m3_encode((double)t);  // t >= 0: an unsigned E4M3
  const float sg = (float)e4m3_decode(sbyte) * g;
  const float r = sg > 0.f ? 1.0f / sg : 0.f;
  for (int i = 0; i < n; ++i) {
    const float y = (float)x[i] * r;
    const uint8_t c = e2m1_encode((double)y);
    if (codes) codes[i] = c;
    if (deq) deq[i] = e2m1_decode(c) * e4m3_decode(sbyte) * (double)g;
  }
  return sbyte;
}

/* Dequantised NVFP4 form of one (document, head) slice: [L][d], per token,
 * 16-channel blocks. */
void nv_form(const double* x, int s, int L, int h, int H, int d, float g, std::vector<double>& out) {
  std::vector<double> xs;
  slice_n(x, s, L, h, H, d, xs);
  out.assign((size_t)L * d, 0.0);
  for (int j = 0; j < L; ++j)
    for (int c0 = 0; c0 < d; c0 += 16)
      nv_quant_block(&xs[(size_t)j * d + c0], 16, g, nullptr, &out[(size_t)j * d + c0]);
}

/* The mixed path's option: S from NVFP4 Q and K with decode scales gq, gk. */
struct NvOpt {
  bool on;
  float gq, gk;
};

/* Rule L operand selection: per-token form on the diagonal block, token-block
 * form elsewhere. */
inline const double* pick(const std::vector<double>& tb, const std::vector<double>& pt, int lj,
                          int li, int d) {
  return ((lj >> 5) == (li >> 5)) ? &pt[(size_t)lj * d] : &tb[(size_t)lj * d];
}

/* Quantise a row vector p[0..n) in 32-blocks along its index (doc-local
 * blocks), in place, when enabled. */
void quant_along(std::vector<double>& p, int n, bool on, int rule) {
  if (!on) return;
  for (int b0 = 0; b0 < n; b0 += 32) {
    const int nb = std::min(32, n - b0);
    quant_block(&p[b0], nb, 1, nullptr, 0, &p[b0], 1, rule);
  }
}

/* flags of the MXFP8 emulation.  MX_QUANT_P is the method; the others are
 * accuracy-study switches that each take one quantisation out (or, for
 * MX_SYM_GUARD, apply the per-token guard to the query side of dK and dV). */
enum {
  MX_QUANT_P = 1,     // quantise the computed P and dS operands (the method's rule)
  MX_RULE_OCP = 2,    // use RULE_OCP for every scale instead of RULE_RCEIL
  MX_KEEP_INPUTS = 4, // study: Q, K, V, dO unquantised
  MX_KEEP_P = 8,      // study: P~ (forward) and P~T (backward) unquantised
  MX_KEEP_DS = 16,    // study: dS~ and dS~T unquantised
  MX_SYM_GUARD = 32   // study: Q and dO per token on the diagonal query block of dK, dV
};
inline int rule_of(int flags) { return (flags & MX_RULE_OCP) ? RULE_OCP : RULE_RCEIL; }
inline bool quant_p(int flags) { return (flags & MX_QUANT_P) && !(flags & MX_KEEP_P); }
inline bool quant_ds(int flags) { return (flags & MX_QUANT_P) && !(flags & MX_KEEP_DS); }

/* P~ of the forward: the row's probabilities are quantised in the form
 *   u_ij = 2^(S_ij log2(e) - M_i),  M_i = ceil(max_j S_ij log2(e)),
 * i.e. exp(S_ij) up to an integer power of two.  Because an MX block is
 * quantised relative to its own power-of-two scale, every integer reference
 * M_i yields the same codes; a single-pass (online-softmax) kernel whose
 * running reference is an integer power of two therefore produces exactly
 * these codes.  O_i = sum_j u~_ij V~_j / sum_j u_ij (the row sum is taken
 * before quantisation).  Without MX_QUANT_P this is the ordinary softmax. */
void fwd_p_tilde(const std::vector<double>& srow, int n, bool on, int rule,
                 std::vector<double>& pq) {
  const double LOG2E = 1.4426950408889634074;
  double mx = -INFINITY;
  for (int j = 0; j < n; ++j) mx = std::max(mx, srow[j] * LOG2E);
  const double M = std::ceil(mx);
  pq.resize(n);
  double l = 0.0;
  for (int j = 0; j < n; ++j) {
    pq[j] = std::exp2(srow[j] * LOG2E - M);
    l += pq[j];
  }
  quant_along(pq, n, on, rule);
  for (int j = 0; j < n; ++j) pq[j] /= l;
}

/* Quantised score row: S_ij = scale * sum_r Qpt_ir * K~_jr with K~ picked by
 * rule L; returns normalised fp64 P (p), max m and sum l. */
int mx_score_row(const double* qi_pt, const std::vector<double>& Ktb,
                 const std::vector<double>& Kpt, int li, int d, double scale,
                 std::vector<double>& srow, std::vector<double>& p, double& m, double& l) {
  const int n = li + 1;
  srow.assign(n, 0.0);
  for (int j = 0; j < n; ++j) {
    const double* kj = pick(Ktb, Kpt, j, li, d);
    double acc = 0.0;
    for (int r = 0; r < d; ++r) acc += qi_pt[r] * kj[r];
    srow[j] = acc * scale;
  }
  m = -INFINITY;
  for (int j = 0; j < n; ++j) m = std::max(m, srow[j]);
  p.resize(n);
  l = 0.0;
  for (int j = 0; j < n; ++j) {
    p[j] = std::exp(srow[j] - m);
    l += p[j];
  }
  for (int j = 0; j < n; ++j) p[j] /= l;
  return n;
}

}  // namespace

extern "C" {

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Exact forward.  q [T][Hq][d], k/v [T][Hkv][d], o [T][Hq][d], lse [Hq][T].
 * Rows of zero-length documents do not exist; every row sees its diagonal. */
void orc_attn_fwd(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                  const double* q, const double* k, const double* v, double* o, double* lse) {
  const Problem P{T, nd, Hq, Hkv, d, cu, scale};
  const std::vector<Task> tasks = head_doc_tasks(P, Hq);
#pragma omp parallel for schedule(dynamic, 1)
  for (long ti = 0; ti < (long)tasks.size(); ++ti) fwd_doc_head(P, tasks[ti].doc, tasks[ti].h, q, k, v, o, lse);
}

/* Exact backward (and forward).  Writes o, lse, dq [T][Hq][d] and
 * dk, dv [T][Hkv][d].  D uses the oracle's own fp64 O.  One task per
 * (document, kv head) accumulates dK and dV privately in a fixed order
 * (query heads of the group ascending, query rows ascending). */
void orc_attn_bwd(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                  const double* q, const double* k, const double* v, const double* dout,
                  double* o, double* lse, double* dq, double* dk, double* dv) {
  const Problem P{T, nd, Hq, Hkv, d, cu, scale};
  const int G = P.G();
  const std::vector<Task> tasks = head_doc_tasks(P, Hkv);
#pragma omp parallel for schedule(dynamic, 1)
  for (long ti = 0; ti < (long)tasks.size(); ++ti) {
    const int kdoc = tasks[ti].doc, g = tasks[ti].h;
    const int s = cu[kdoc], L = cu[kdoc + 1] - cu[kdoc];
    std::vector<double> Kt, Vt, Kn, srow, p, dp, orow(d), dqrow(d);
    slice_t(k, s, L, g, Hkv, d, Kt);
    slice_t(v, s, L, g, Hkv, d, Vt);
    slice_n(k, s, L, g, Hkv, d, Kn);
    std::vector<double> Vn;
    slice_n(v, s, L, g, Hkv, d, Vn);
    std::vector<double> dK((size_t)L * d, 0.0), dV((size_t)L * d, 0.0);
    for (int h = g * G; h < (g + 1) * G; ++h) {
      for (int li = 0; li < L; ++li) {
        const int i = s + li;
        const double* qi = &q[idx3(i, h, 0, Hq, d)];
        const double* doi = &dout[idx3(i, h, 0, Hq, d)];
        double m, l;
        const int n = score_row(qi, Kt, L, d, li, scale, srow, p, m, l);
        // forward row: O_i = sum_j P_ij V_j
        std::fill(orow.begin(), orow.end(), 0.0);
        for (int j = 0; j < n; ++j)
          for (int r = 0; r < d; ++r) orow[r] += p[j] * Vn[(size_t)j * d + r];
        for (int r = 0; r < d; ++r) o[idx3(i, h, r, Hq, d)] = orow[r];
        lse[(size_t)h * T + i] = m + std::log(l);
        // D_i = dO_i . O_i
        double D = 0.0;
        for (int r = 0; r < d; ++r) D += doi[r] * orow[r];
        // dP_ij = dO_i . V_j (summed over r in order), dS_ij = P_ij (dP_ij - D_i)
        dp.assign(n, 0.0);
        for (int r = 0; r < d; ++r) {
          const double dr = doi[r];
          const double* vr = &Vt[(size_t)r * L];
          for (int j = 0; j < n; ++j) dp[j] += dr * vr[j];
        }
        std::fill(dqrow.begin(), dqrow.end(), 0.0);
        for (int j = 0; j < n; ++j) {
          const double ds = p[j] * (dp[j] - D);
          const double* kj = &Kn[(size_t)j * d];
          double* dkj = &dK[(size_t)j * d];
          double* dvj = &dV[(size_t)j * d];
          for (int r = 0; r < d; ++r) {
            dqrow[r] += ds * kj[r];
            dkj[r] += ds * qi[r];
            dvj[r] += p[j] * doi[r];
          }
        }
        for (int r = 0; r < d; ++r) dq[idx3(i, h, r, Hq, d)] = scale * dqrow[r];
      }
    }
    for (int j = 0; j < L; ++j)
      for (int r = 0; r < d; ++r) {
        dk[idx3(s + j, g, r, Hkv, d)] = scale * dK[(size_t)j * d + r];
        dv[idx3(s + j, g, r, Hkv, d)] = dV[(size_t)j * d + r];
      }
  }
}

/* Exact O, LSE and dQ of selected (token, query head) rows, each computed on
 * its own (the row needs only its own document's keys).  o/dq: [n][d], lse [n]. */
void orc_attn_rows(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                   const double* q, const double* k, const double* v, const double* dout, int n,
                   const int32_t* tok, const int32_t* head, double* o, double* lse, double* dq) {
  const Problem P{T, nd, Hq, Hkv, d, cu, scale};
  const int G = P.G();
#pragma omp parallel for schedule(dynamic, 1)
  for (int si = 0; si < n; ++si) {
    const int i = tok[si], h = head[si], g = h / G;
    const int kdoc = (int)(std::upper_bound(cu, cu + nd + 1, i) - cu) - 1;
    const int s = cu[kdoc], li = i - s;
    const int L = li + 1;  // only keys s..i are needed
    std::vector<double> Kt, Kn, Vn, srow, p;
    slice_t(k, s, L, g, Hkv, d, Kt);
    slice_n(k, s, L, g, Hkv, d, Kn);
    slice_n(v, s, L, g, Hkv, d, Vn);
    const double* qi = &q[idx3(i, h, 0, Hq, d)];
    const double* doi = &dout[idx3(i, h, 0, Hq, d)];
    double m, l;
    const int nn = score_row(qi, Kt, L, d, li, scale, srow, p, m, l);
    std::vector<double> orow(d, 0.0), dqrow(d, 0.0);
    for (int j = 0; j < nn; ++j)
      for (int r = 0; r < d; ++r) orow[r] += p[j] * Vn[(size_t)j * d + r];
    double D = 0.0;
    for (int r = 0; r < d; ++r) D += doi[r] * orow[r];
    for (int j = 0; j < nn; ++j) {
      double dpj = 0.0;
      for (int r = 0; r < d; ++r) dpj += doi[r] * Vn[(size_t)j * d + r];
      const double ds = p[j] * (dpj - D);
      for (int r = 0; r < d; ++r) dqrow[r] += ds * Kn[(size_t)j * d + r];
    }
    for (int r = 0; r < d; ++r) {
      o[(size_t)si * d + r] = orow[r];
      dq[(size_t)si * d + r] = scale * dqrow[r];
    }
    lse[si] = m + std::log(l);
  }
}

/* Exact dK and dV of selected (token, kv head) keys: every query row i >= j of
 * the key's document, for every query head of the group, is recomputed in
 * full (its own O_i and D_i).  dk/dv: [n][d]. */
void orc_attn_kv_cols(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                      const double* q, const double* k, const double* v, const double* dout,
                      int n, const int32_t* tok, const int32_t* kvhead, double* dk, double* dv) {
  const Problem P{T, nd, Hq, Hkv, d, cu, scale};
  const int G = P.G();
#pragma omp parallel for schedule(dynamic, 1)
  for (int si = 0; si < n; ++si) {
    const int j = tok[si], g = kvhead[si];
    const int kdoc = (int)(std::upper_bound(cu, cu + nd + 1, j) - cu) - 1;
    const int s = cu[kdoc], e = cu[kdoc + 1], L = e - s, lj = j - s;
    std::vector<double> Kt, Vn, srow, p, orow(d);
    slice_t(k, s, L, g, Hkv, d, Kt);
    slice_n(v, s, L, g, Hkv, d, Vn);
    std::vector<double> dkj(d, 0.0), dvj(d, 0.0);
    for (int h = g * G; h < (g + 1) * G; ++h) {
      for (int li = lj; li < L; ++li) {
        const int i = s + li;
        const double* qi = &q[idx3(i, h, 0, Hq, d)];
        const double* doi = &dout[idx3(i, h, 0, Hq, d)];
        double m, l;
        const int nn = score_row(qi, Kt, L, d, li, scale, srow, p, m, l);
        std::fill(orow.begin(), orow.end(), 0.0);
        for (int jj = 0; jj < nn; ++jj)
          for (int r = 0; r < d; ++r) orow[r] += p[jj] * Vn[(size_t)jj * d + r];
        double D = 0.0;
        for (int r = 0; r < d; ++r) D += doi[r] * orow[r];
        double dpj = 0.0;
        for (int r = 0; r < d; ++r) dpj += doi[r] * Vn[(size_t)lj * d + r];
        const double ds = p[lj] * (dpj - D);
        for (int r = 0; r < d; ++r) {
          dkj[r] += ds * qi[r];
          dvj[r] += p[lj] * doi[r];
        }
      }
    }
    for (int r = 0; r < d; ++r) {
      dk[(size_t)si * d + r] = scale * dkj[r];
      dv[(size_t)si * d + r] = dvj[r];
    }
  }
}

/* Exact dK and dV of selected (token, kv head) keys from the exact forward
 * rows of the queries that see them: o [T][Hq][d] and lse [Hq][T] must hold
 * the exact O_i and LSE_i of every query i >= j of key j's document for the
 * query heads of its group (other entries are not read).  Same sums as
 * orc_attn_kv_cols, with P_ij = exp(S_ij - LSE_i) (the normalised softmax, by
 * the definition of LSE) and D_i = dO_i . O_i, so no query row is recomputed.
 * dk/dv: [n][d]. */
void orc_attn_kv_cols_from_rows(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                                const double* q, const double* k, const double* v, const double* dout,
                                const double* o, const double* lse, int n, const int32_t* tok,
                                const int32_t* kvhead, double* dk, double* dv) {
  const Problem P{T, nd, Hq, Hkv, d, cu, scale};
  const int G = P.G();
#pragma omp parallel for schedule(dynamic, 1)
  for (int si = 0; si < n; ++si) {
    const int j = tok[si], g = kvhead[si];
    const int kdoc = (int)(std::upper_bound(cu, cu + nd + 1, j) - cu) - 1;
    const int e = cu[kdoc + 1];
    const double* kj = &k[idx3(j, g, 0, Hkv, d)];
    const double* vj = &v[idx3(j, g, 0, Hkv, d)];
    std::vector<double> dkj(d, 0.0), dvj(d, 0.0);
    for (int h = g * G; h < (g + 1) * G; ++h) {
      for (int i = j; i < e; ++i) {
        const double* qi = &q[idx3(i, h, 0, Hq, d)];
        const double* doi = &dout[idx3(i, h, 0, Hq, d)];
        const double* oi = &o[idx3(i, h, 0, Hq, d)];
        double sij = 0.0, dpj = 0.0, D = 0.0;
        for (int r = 0; r < d; ++r) {
          sij += qi[r] * kj[r];
          dpj += doi[r] * vj[r];
          D += doi[r] * oi[r];
        }
        const double pij = std::exp(scale * sij - lse[(size_t)h * T + i]);
        const double ds = pij * (dpj - D);
        for (int r = 0; r < d; ++r) {
          dkj[r] += ds * qi[r];
          dvj[r] += pij * doi[r];
        }
      }
    }
    for (int r = 0; r < d; ++r) {
      dk[(size_t)si * d + r] = scale * dkj[r];
      dv[(size_t)si * d + r] = dvj[r];
    }
  }
}

/* ---- MXFP8 quantiser -------------------------------------------------- */

uint8_t orc_e4m3_encode(double y) { return e4m3_encode(y); }
double orc_e4m3_decode(uint8_t c) { return e4m3_decode(c); }
int orc_block_exponent(double amax, int rule) { return block_exponent(amax, rule); }

/* Quantise one block of n values (stride 1).  Returns the scale byte. */
uint8_t orc_quant_block(const double* x, int n, uint8_t* codes, double* deq, int rule) {
  return quant_block(x, n, 1, codes, 1, deq, 1, rule);
}

/* quantize_mxfp8 of a bf16-valued [T][H][d] tensor (given as exact doubles),
 * with scale rule `rule` (RULE_RCEIL = 0, RULE_OCP = 1).
 * forms bit 0: token-block form -- codes val_tb [T][H][d] and scales
 *   scale_tb [T/32 + n_docs][H][d/32], block m of document k at slot
 *   floor(s_k/32) + k + m; slots that hold no block are left untouched.
 * forms bit 1: per-token form -- codes val_pt [T][H][d], scales
 *   scale_pt [T][H][d/32]. */
void orc_quantize_mxfp8(const double* x, int T, int H, int d, const int32_t* cu, int nd,
                        int forms, int rule, uint8_t* val_tb, uint8_t* scale_tb,
                        uint8_t* val_pt, uint8_t* scale_pt) {
  const int nG = d / 32;
  if (forms & 2) {
#pragma omp parallel for schedule(static)
    for (long t = 0; t < (long)T; ++t)
      for (int h = 0; h < H; ++h)
        for (int gi = 0; gi < nG; ++gi) {
          const size_t o = idx3((int)t, h, gi * 32, H, d);
          scale_pt[((size_t)t * H + h) * nG + gi] =
              quant_block(&x[o], 32, 1, &val_pt[o], 1, nullptr, 0, rule);
        }
  }
  if (forms & 1) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int k = 0; k < nd; ++k) {
      const int s = cu[k], L = cu[k + 1] - cu[k];
      for (int m = 0; 32 * m < L; ++m) {
        const int t0 = s + 32 * m, nb = std::min(32, L - 32 * m);
        const size_t slot = (size_t)(s / 32) + k + m;
        for (int h = 0; h < H; ++h)
          for (int gi = 0; gi < nG; ++gi) {
            double amax = 0.0;
            for (int t = t0; t < t0 + nb; ++t)
              for (int c = 0; c < 32; ++c)
                amax = std::max(amax, std::fabs(x[idx3(t, h, gi * 32 + c, H, d)]));
            const int X = block_exponent(amax, rule);
            for (int t = t0; t < t0 + nb; ++t)
              for (int c = 0; c < 32; ++c) {
                const size_t o = idx3(t, h, gi * 32 + c, H, d);
                val_tb[o] = e4m3_encode(std::ldexp(x[o], -X));
              }
            scale_tb[(slot * H + h) * nG + gi] = (uint8_t)(X + 127);
          }
      }
    }
  }
}

/* ---- MXFP8 attention emulation (rule L) --------------------------------- */

/* Forward of the emulation: S from Q~pt and K~ (rule L); P~ quantised per
 * (row, key block) in the integer-power-of-two form of fwd_p_tilde when
 * flags & MX_QUANT_P; O = sum_j P~_ij V~_j (rule L); LSE from the quantised
 * S.  Every scale uses rule_of(flags). */
}  // extern "C"

namespace {

void mx_attn_fwd(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                 const double* q, const double* k, const double* v, int flags, const NvOpt& nv,
                 double* o, double* lse) {
  const Problem P{T, nd, Hq, Hkv, d, cu, scale};
  const std::vector<Task> tasks = head_doc_tasks(P, Hq);
  const bool qp = quant_p(flags), ex = flags & MX_KEEP_INPUTS;
  const int rule = rule_of(flags);
#pragma omp parallel for schedule(dynamic, 1)
  for (long ti = 0; ti < (long)tasks.size(); ++ti) {
    const int kdoc = tasks[ti].doc, h = tasks[ti].h, g = h / P.G();
    const int s = cu[kdoc], L = cu[kdoc + 1] - cu[kdoc];
    std::vector<double> Qtb, Qpt, Ktb, Kpt, Vtb, Vpt, srow, p, pq, orow(d);
    mx_forms(q, s, L, h, Hq, d, rule, Qtb, Qpt, ex);
    mx_forms(k, s, L, g, Hkv, d, rule, Ktb, Kpt, ex);
    mx_forms(v, s, L, g, Hkv, d, rule, Vtb, Vpt, ex);
    // the scores' operands: Q~pt and K~ by rule L, or NVFP4 Q and K (mixed path)
    std::vector<double> Qs, Ks;
    if (nv.on) {
      nv_form(q, s, L, h, Hq, d, nv.gq, Qs);
      nv_form(k, s, L, g, Hkv, d, nv.gk, Ks);
    }
    for (int li = 0; li < L; ++li) {
      double m, l;
      const int n = nv.on ? mx_score_row(&Qs[(size_t)li * d], Ks, Ks, li, d, scale, srow, p, m, l)
                          : mx_score_row(&Qpt[(size_t)li * d], Ktb, Kpt, li, d, scale, srow, p, m, l);
      fwd_p_tilde(srow, n, qp, rule, pq);
      std::fill(orow.begin(), orow.end(), 0.0);
      for (int j = 0; j < n; ++j) {
        const double* vj = pick(Vtb, Vpt, j, li, d);
        for (int r = 0; r < d; ++r) orow[r] += pq[j] * vj[r];
      }
      for (int r = 0; r < d; ++r) o[idx3(s + li, h, r, Hq, d)] = orow[r];
      lse[(size_t)h * T + s + li] = m + std::log(l);
    }
  }
}

/* Backward of the emulation: the straight-through gradient of the emulated
 * forward, from the same quantised operands.  Writes o, lse (the emulated
 * forward), dq [T][Hq][d], dk/dv [T][Hkv][d].  P below is the normalised
 * fp64 softmax exp(S - LSE) of the quantised scores (a backward recomputes it
 * from the saved LSE); every scale uses rule_of(flags).
 *   D_i   = dO_i . O_i        (bf16 dO, emulated O)
 *   dP_ij = dO~pt_i . V~_j    (V~ by rule L)
 *   dS_ij = P_ij (dP_ij - D_i) in fp64
 *   dQ_i  = scale sum_j dS~_ij K~_j            (dS~ per (row, key block))
 *   dK_j  = scale sum_i dS~T_ji Q~tb_i         (dS~T per (key, query block))
 *   dV_j  =       sum_i P~T_ji dO~tb_i         (P~T per (key, query block)) */
void mx_attn_bwd(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                 const double* q, const double* k, const double* v, const double* dout, int flags,
                 const NvOpt& nv, double* o, double* lse, double* dq, double* dk, double* dv) {
  const Problem P{T, nd, Hq, Hkv, d, cu, scale};
  const int G = P.G();
  const bool qp = quant_p(flags), qds = quant_ds(flags), ex = flags & MX_KEEP_INPUTS;
  const bool sym = flags & MX_SYM_GUARD;
  const int rule = rule_of(flags);
  const std::vector<Task> tasks = head_doc_tasks(P, Hkv);
#pragma omp parallel for schedule(dynamic, 1)
  for (long ti = 0; ti < (long)tasks.size(); ++ti) {
    const int kdoc = tasks[ti].doc, g = tasks[ti].h;
    const int s = cu[kdoc], L = cu[kdoc + 1] - cu[kdoc];
    std::vector<double> Ktb, Kpt, Vtb, Vpt, Qtb, Qpt, dOtb, dOpt, srow, p, pq, orow(d), Qs, Ks;
    mx_forms(k, s, L, g, Hkv, d, rule, Ktb, Kpt, ex);
    mx_forms(v, s, L, g, Hkv, d, rule, Vtb, Vpt, ex);
    if (nv.on) nv_form(k, s, L, g, Hkv, d, nv.gk, Ks);
    std::vector<double> dK((size_t)L * d, 0.0), dV((size_t)L * d, 0.0);
    for (int h = g * G; h < (g + 1) * G; ++h) {
      mx_forms(q, s, L, h, Hq, d, rule, Qtb, Qpt, ex);
      mx_forms(dout, s, L, h, Hq, d, rule, dOtb, dOpt, ex);
      if (nv.on) nv_form(q, s, L, h, Hq, d, nv.gq, Qs);
      // rows are processed in 32-row query blocks so that P^T and dS^T can be
      // quantised per (key row, query block)
      for (int b0 = 0; b0 < L; b0 += 32) {
        const int nb = std::min(32, L - b0);
        const int ncol = b0 + nb;  // keys 0..ncol-1 can be visible to this block
        std::vector<double> Pblk((size_t)nb * ncol, 0.0), dSblk((size_t)nb * ncol, 0.0);
        for (int a = 0; a < nb; ++a) {
          const int li = b0 + a, i = s + li;
          double m, l;
          // the same scores as the forward's (NVFP4 Q and K on the mixed path)
          const int n = nv.on ? mx_score_row(&Qs[(size_t)li * d], Ks, Ks, li, d, scale, srow, p, m, l)
                              : mx_score_row(&Qpt[(size_t)li * d], Ktb, Kpt, li, d, scale, srow, p, m, l);
          fwd_p_tilde(srow, n, qp, rule, pq);
          std::fill(orow.begin(), orow.end(), 0.0);
          for (int j = 0; j < n; ++j) {
            const double* vj = pick(Vtb, Vpt, j, li, d);
            for (int r = 0; r < d; ++r) orow[r] += pq[j] * vj[r];
          }
          for (int r = 0; r < d; ++r) o[idx3(i, h, r, Hq, d)] = orow[r];
          lse[(size_t)h * T + i] = m + std::log(l);
          const double* doi = &dout[idx3(i, h, 0, Hq, d)];
          double D = 0.0;
          for (int r = 0; r < d; ++r) D += doi[r] * orow[r];
          std::vector<double> ds(n);
          for (int j = 0; j < n; ++j) {
            const double* vj = pick(Vtb, Vpt, j, li, d);
            double dpj = 0.0;
            for (int r = 0; r < d; ++r) dpj += dOpt[(size_t)li * d + r] * vj[r];
            ds[j] = p[j] * (dpj - D);
            Pblk[(size_t)a * ncol + j] = p[j];
            dSblk[(size_t)a * ncol + j] = ds[j];
          }
          // dQ_i = scale sum_j dS~_ij K~_j
          std::vector<double> dsq(ds);
          quant_along(dsq, n, qds, rule);
          std::vector<double> dqrow(d, 0.0);
          for (int j = 0; j < n; ++j) {
            const double* kj = pick(Ktb, Kpt, j, li, d);
            for (int r = 0; r < d; ++r) dqrow[r] += dsq[j] * kj[r];
          }
          for (int r = 0; r < d; ++r) dq[idx3(i, h, r, Hq, d)] = scale * dqrow[r];
        }
        // dK, dV: columns of this query block, quantised per (key, query block)
        std::vector<double> pc(nb), dc(nb);
        for (int j = 0; j < ncol; ++j) {
          for (int a = 0; a < nb; ++a) {
            pc[a] = Pblk[(size_t)a * ncol + j];
            dc[a] = dSblk[(size_t)a * ncol + j];
          }
          if (qp) quant_block(pc.data(), nb, 1, nullptr, 0, pc.data(), 1, rule);
          if (qds) quant_block(dc.data(), nb, 1, nullptr, 0, dc.data(), 1, rule);
          double* dkj = &dK[(size_t)j * d];
          double* dvj = &dV[(size_t)j * d];
          for (int a = 0; a < nb; ++a) {
            const int li = b0 + a;
            if (li < j) continue;  // masked: exactly zero
            // query-side operands of the query contraction: token-block form
            // in every query block (every query with a non-zero term here is
            // causally after key j, so no guard is needed)
            const bool pt_side = sym && (li >> 5) == (j >> 5);
            const double* qi = pt_side ? &Qpt[(size_t)li * d] : &Qtb[(size_t)li * d];
            const double* doi = pt_side ? &dOpt[(size_t)li * d] : &dOtb[(size_t)li * d];
            for (int r = 0; r < d; ++r) {
              dkj[r] += dc[a] * qi[r];
              dvj[r] += pc[a] * doi[r];
            }
          }
        }
      }
    }
    for (int j = 0; j < L; ++j)
      for (int r = 0; r < d; ++r) {
        dk[idx3(s + j, g, r, Hkv, d)] = scale * dK[(size_t)j * d + r];
        dv[idx3(s + j, g, r, Hkv, d)] = dV[(size_t)j * d + r];
      }
  }
}

}  // namespace

extern "C" {

void orc_mx_attn_fwd(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                     const double* q, const double* k, const double* v, int flags, double* o,
                     double* lse) {
  mx_attn_fwd(T, nd, cu, Hq, Hkv, d, scale, q, k, v, flags, NvOpt{false, 1.f, 1.f}, o, lse);
}

void orc_mx_attn_bwd(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                     const double* q, const double* k, const double* v, const double* dout,
                     int flags, double* o, double* lse, double* dq, double* dk, double* dv) {
  mx_attn_bwd(T, nd, cu, Hq, Hkv, d, scale, q, k, v, dout, flags, NvOpt{false, 1.f, 1.f}, o, lse, dq,
              dk, dv);
}

/* ---- mixed NVFP4/FP8 path ------------------------------------------------ */

uint8_t orc_e2m1_encode(double y) { return e2m1_encode(y); }
double orc_e2m1_decode(uint8_t c) { return e2m1_decode(c); }

/* One NVFP4 block of n values with decode scale g: codes (one per value),
 * dequantised values; returns the E4M3 scale byte. */
uint8_t orc_nv_quant_block(const double* x, int n, float g, uint8_t* codes, double* deq) {
  return nv_quant_block(x, n, g, codes, deq);
}

/* NVFP4 of a bf16-valued [T][H][d] tensor (exact doubles), decode scale g:
 * codes [T][H][d/2] (channel 2i in the low nibble of byte i, 2i + 1 in the
 * high nibble), scales [T][H][d/16]. */
void orc_quantize_nvfp4(const double* x, int T, int H, int d, float g, uint8_t* codes, uint8_t* scales) {
#pragma omp parallel for schedule(static)
  for (long t = 0; t < (long)T; ++t)
    for (int h = 0; h < H; ++h)
      for (int b = 0; b < d / 16; ++b) {
        uint8_t c[16];
        const size_t o = idx3((int)t, h, 16 * b, H, d);
        scales[((size_t)t * H + h) * (d / 16) + b] = nv_quant_block(&x[o], 16, g, c, nullptr);
        for (int i = 0; i < 8; ++i) codes[o / 2 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
      }
}

/* The mixed path's forward and backward: the MXFP8 emulation with the scores
 * taken from NVFP4 Q and K (decode scales gq, gk), in both passes. */
void orc_nvmx_attn_fwd(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                       const double* q, const double* k, const double* v, int flags, float gq, float gk,
                       double* o, double* lse) {
  mx_attn_fwd(T, nd, cu, Hq, Hkv, d, scale, q, k, v, flags, NvOpt{true, gq, gk}, o, lse);
}

void orc_nvmx_attn_bwd(int T, int nd, const int32_t* cu, int Hq, int Hkv, int d, double scale,
                       const double* q, const double* k, const double* v, const double* dout,
                       int flags, float gq, float gk, double* o, double* lse, double* dq, double* dk,
                       double* dv) {
  mx_attn_bwd(T, nd, cu, Hq, Hkv, d, scale, q, k, v, dout, flags, NvOpt{true, gq, gk}, o, lse, dq, dk,
              dv);
}

}  // extern "C"
