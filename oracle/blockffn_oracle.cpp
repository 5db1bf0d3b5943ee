// BlockFFN chunk-layer oracle: plain, slow, fp64, on the CPU.
//
// TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the benchmark's CPU-baseline
// leg may load this library. It shares no code, header, table or helper with the CUDA path; the
// two meet only through the seeded input generator.
//
// What it computes, per token t of a chunk of L consecutive tokens (the BlockFFN layer as the
// pages describe it; the pages print no equations, so each step names the passage it restates):
//   s_{t,i} = sum_k x_{t,k} Wr[k,i] + b_i                     router projection
//   a_{t,i} = max(s_{t,i}, 0)                                 ReLU  (lsdiaocha.cn BlockFFN article, section 2:
//                                                             the router combines a ReLU activation with an RMSNorm layer)
//   r_{t,i} = g_i a_{t,i} / sqrt((1/E) sum_i a_{t,i}^2)       RMSNorm over the E router outputs (same
//                                                             passage, and the BlockFFN abstract, which names a
//                                                             router built from ReLU followed by RMSNorm); r_t = 0
//                                                             when every a is 0
//   E_i(x) = W2_i Swish(W1_i x), Swish(u) = u / (1 + e^-u)    non-gated MLP expert with Swish (article, section 2)
//   y_t = sum_i r_{t,i} E_i(x_t)                              router-weighted combination; the mask of
//                                                             section 4 removes the terms with r = 0
// Active sets: A_t = {i : s_{t,i} > 0}; the chunk's union U = U_t A_t (article, section 4: the union of
// the experts the candidate tokens activate); token-level sparsity counts the (t,i) with i not in A_t,
// chunk-level sparsity counts the experts outside U (article, section 1; BlockFFN abstract).
//
// Readings where the pages are silent: RMSNorm has no epsilon (a token with no active expert gets
// r = 0 and y = 0); Swish has beta = 1; the RMSNorm mean runs over all E entries, zeros included;
// the union is listed in ascending expert order.
//
// The ReMoE router variant (intelliparadigm survey, section 5.1: the gate G = ReLU(x W_g) and the layer's
// output the sum of G_i times expert i, divided by the sum of G): norm = 1 replaces the RMS by the sum of
// the ReLU outputs, r_{t,i} = g_i a_{t,i} / sum_i a_{t,i} (r_t = 0 when every a is 0); the gain g is kept
// (g = 1 gives the survey's formula).
//
// The CLS-aware training objectives (activation locality, chunk sparsification; article, section 3) and
// their backward through the router, the fp8 weight quantiser, and the layer's own backward are at the end
// of this file, with the readings they take.
//
// Storage: x is bf16 bit patterns [L,d]; Wr fp32 [d,E]; br fp32 [E] (may be null = no bias);
// g fp32 [E]; W1 bf16 bits [E,de,d]; W2 bf16 bits [E,d,de]; everything row-major.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// Planted mistakes, used only by the tests that check each pin can fail (0 = the correct oracle).
int g_mutation = 0;

double widen_bf16(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

double swish(double u) {
  if (g_mutation == 2) return u / (1.0 + std::exp(u));  // planted: wrong sign in the sigmoid
  return u / (1.0 + std::exp(-u));
}

// Router for one token: s (pre-activation), r (normalised weights), active flags.
void router_token(const uint16_t* xt, int d, const float* Wr, const float* br, const float* g,
                  int E, int norm, double* s, double* r, uint8_t* act) {
  for (int i = 0; i < E; ++i) {
    double acc = 0.0;
    for (int k = 0; k < d; ++k) {
      int kk = (g_mutation == 4) ? (d - 1 - k) : k;  // planted: reversed router input index
      acc += widen_bf16(xt[kk]) * static_cast<double>(Wr[static_cast<size_t>(k) * E + i]);
    }
    if (br != nullptr && g_mutation != 1) acc += static_cast<double>(br[i]);  // planted 1: bias dropped
    s[i] = acc;
  }
  double sumsq = 0.0, sum = 0.0;
  int n_pos = 0;
  for (int i = 0; i < E; ++i) {
    double a = s[i] > 0.0 ? s[i] : 0.0;
    sumsq += a * a;
    sum += a;
    if (a > 0.0) ++n_pos;
  }
  // planted 3: mean over the active entries only instead of over all E
  double denom = (g_mutation == 3) ? static_cast<double>(n_pos > 0 ? n_pos : 1) : static_cast<double>(E);
  double ms = sumsq / denom;
  // the normaliser: the RMS of the ReLU outputs (BlockFFN), or their sum (ReMoE)
  double nrm = std::sqrt(ms);
  if (norm == 1) nrm = (g_mutation == 8) ? sum / static_cast<double>(E) : sum;  // planted 8: the mean, not the sum
  for (int i = 0; i < E; ++i) {
    double a = s[i] > 0.0 ? s[i] : 0.0;
    act[i] = s[i] > 0.0 ? 1 : 0;
    r[i] = (nrm > 0.0) ? static_cast<double>(g[i]) * a / nrm : 0.0;
  }
}

// One expert applied to one token: out[d] = W2_i Swish(W1_i x_t).
void expert_token(const uint16_t* xt, int d, const uint16_t* W1, const uint16_t* W2, int de, int i,
                  double* out) {
  std::vector<double> h(de);
  const uint16_t* W1i = W1 + static_cast<size_t>(i) * de * d;
  const uint16_t* W2i = W2 + static_cast<size_t>(i) * d * de;
  for (int j = 0; j < de; ++j) {
    double u = 0.0;
    for (int k = 0; k < d; ++k) u += widen_bf16(W1i[static_cast<size_t>(j) * d + k]) * widen_bf16(xt[k]);
    h[j] = swish(u);
  }
  for (int k = 0; k < d; ++k) {
    double acc = 0.0;
    for (int j = 0; j < de; ++j) {
      // planted 5: W2 read as if it were stored [de, d]
      size_t idx = (g_mutation == 5) ? static_cast<size_t>(j) * d + k : static_cast<size_t>(k) * de + j;
      acc += widen_bf16(W2i[idx]) * h[j];
    }
    out[k] = acc;
  }
}

void forward_tokens(int t0, int t1, const uint16_t* x, int d, const float* Wr, const float* br,
                    const float* g, const uint16_t* W1, const uint16_t* W2, int E, int de, int sparse, int norm,
                    double* y, double* r_out, uint8_t* act_out) {
  std::vector<double> s(E), r(E), e(d);
  std::vector<uint8_t> act(E);
  for (int t = t0; t < t1; ++t) {
    const uint16_t* xt = x + static_cast<size_t>(t) * d;
    router_token(xt, d, Wr, br, g, E, norm, s.data(), r.data(), act.data());
    double* yt = y + static_cast<size_t>(t) * d;
    for (int k = 0; k < d; ++k) yt[k] = 0.0;
    for (int i = 0; i < E; ++i) {
      if (sparse && !act[i]) continue;  // sparse evaluation: only experts in A_t
      expert_token(xt, d, W1, W2, de, i, e.data());
      for (int k = 0; k < d; ++k) yt[k] += r[i] * e[k];
    }
    if (r_out) for (int i = 0; i < E; ++i) r_out[static_cast<size_t>(t) * E + i] = r[i];
    if (act_out) for (int i = 0; i < E; ++i) act_out[static_cast<size_t>(t) * E + i] = act[i];
  }
}

bool bad_dims(int L, int d, int E, int de) { return L < 0 || d <= 0 || E <= 0 || de <= 0; }

}  // namespace

extern "C" {

void oracle_set_mutation(int m) { g_mutation = m; }
int oracle_get_mutation(void) { return g_mutation; }

double oracle_swish(double u) { return swish(u); }

// Router over a chunk: s, r as fp64 [L,E]; act as 0/1 bytes [L,E].
int oracle_router(const uint16_t* x, int L, int d, const float* Wr, const float* br, const float* g,
                  int E, int norm, double* s, double* r, uint8_t* act) {
  if (bad_dims(L, d, E, 1) || norm < 0 || norm > 1) return 1;
  for (int t = 0; t < L; ++t)
    router_token(x + static_cast<size_t>(t) * d, d, Wr, br, g, E, norm, s + static_cast<size_t>(t) * E,
                 r + static_cast<size_t>(t) * E, act + static_cast<size_t>(t) * E);
  return 0;
}

// Chunk union and sparsity counts from the per-token active flags.
//   active_idx: the experts of U in ascending order (first n_active entries written)
//   tls_zero  : number of (t,i) with i not in A_t
//   cls_zero  : number of experts not in U
int oracle_union(const uint8_t* act, int L, int E, int32_t* active_idx, int32_t* n_active,
                 int64_t* tls_zero, int64_t* cls_zero) {
  if (bad_dims(L, 1, E, 1)) return 1;
  int64_t zeros = 0;
  int n = 0;
  for (int i = 0; i < E; ++i) {
    bool any = false;
    for (int t = 0; t < L; ++t) {
      if (act[static_cast<size_t>(t) * E + i]) any = true;
      else ++zeros;
    }
    if (g_mutation == 6 && i == E - 1) any = false;  // planted: last expert never joins the union
    if (any) active_idx[n++] = i;
  }
  *n_active = n;
  if (tls_zero) *tls_zero = zeros;
  if (cls_zero) *cls_zero = E - n;
  return 0;
}

// Cross-chunk expert reuse (the BlockFFN article, section 5): the number of experts in both of two unions,
// each given as a list of expert indices, counted by marking one list and scanning the other.
int oracle_union_overlap(const int32_t* a, int na, const int32_t* b, int nb, int E, int32_t* overlap) {
  if (E <= 0 || na < 0 || nb < 0) return 1;
  std::vector<uint8_t> in_b(static_cast<size_t>(E), 0);
  for (int q = 0; q < nb; ++q)
    if (b[q] >= 0 && b[q] < E) in_b[b[q]] = 1;
  int hits = 0;
  for (int q = 0; q < na; ++q)
    if (a[q] >= 0 && a[q] < E && in_b[a[q]]) ++hits;
  *overlap = hits;
  return 0;
}

// One expert on one token (exposed for the special-case pins).
int oracle_expert(const uint16_t* xt, int d, const uint16_t* W1, const uint16_t* W2, int de, int i,
                  double* out) {
  if (bad_dims(1, d, 1, de) || i < 0) return 1;
  expert_token(xt, d, W1, W2, de, i, out);
  return 0;
}

// Full layer over one chunk. sparse=0: every expert is evaluated and multiplied by its router
// weight (zero for inactive experts); sparse=1: only the experts of A_t are evaluated.
// y fp64 [L,d]; r_out fp64 [L,E] and act_out [L,E] may be null.
int oracle_chunk_forward(const uint16_t* x, int L, int d, const float* Wr, const float* br,
                         const float* g, const uint16_t* W1, const uint16_t* W2, int E, int de,
                         int sparse, int norm, double* y, double* r_out, uint8_t* act_out) {
  if (bad_dims(L, d, E, de) || norm < 0 || norm > 1) return 1;
  forward_tokens(0, L, x, d, Wr, br, g, W1, W2, E, de, sparse, norm, y, r_out, act_out);
  return 0;
}

// The same over n_tok tokens split across `threads` host threads (tokens are independent, so the
// result is identical to the single-threaded call). Used for the timed CPU baseline.
int oracle_tokens_forward_mt(const uint16_t* x, int n_tok, int d, const float* Wr, const float* br,
                             const float* g, const uint16_t* W1, const uint16_t* W2, int E, int de,
                             int sparse, int norm, int threads, double* y) {
  if (bad_dims(n_tok, d, E, de) || threads < 1 || norm < 0 || norm > 1) return 1;
  std::vector<std::thread> pool;
  for (int w = 0; w < threads; ++w) {
    int t0 = static_cast<int>(static_cast<int64_t>(n_tok) * w / threads);
    int t1 = static_cast<int>(static_cast<int64_t>(n_tok) * (w + 1) / threads);
    if (g_mutation == 7) t1 = t0 + n_tok / threads;  // planted: ranges that drop the remainder tokens
    pool.emplace_back(forward_tokens, t0, t1, x, d, Wr, br, g, W1, W2, E, de, sparse, norm, y,
                      static_cast<double*>(nullptr), static_cast<uint8_t*>(nullptr));
  }
  for (auto& th : pool) th.join();
  return 0;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------------
// CLS-aware training objectives (lsdiaocha.cn BlockFFN article, section 3) and their backward through the
// router, in fp64.  The pages describe both objectives in words only; the readings taken here:
//   p_{t,i} = sigmoid(alpha s_{t,i})              the "sharp sigmoid" that approximates the activation
//                                                 pattern 1[s > 0] (alpha large)
//   activation locality: the binary cross-entropy between each token's approximate pattern and the next
//     token's (the LeftShift of p along the chunk), both soft and both carrying gradient, averaged over
//     the chunks' (L - 1) E adjacent pairs:  L_AL = mean_{c, t < L-1, i} BCE(p_{c,t,i}; q = p_{c,t+1,i})
//     with BCE(p; q) = -(q log p + (1 - q) log(1 - p))
//   chunk sparsification: the probability that at least one token of the chunk activates expert i,
//     averaged over chunks and experts:  L_CS = mean_{c,i} (1 - prod_t (1 - p_{c,t,i}))
// and the combined objective J = w_al L_AL + w_cs L_CS.  Gradients (the plain chain rule):
//   dJ/ds_{c,t,i} = w_al alpha (p_t - p_{t+1}) / N_AL [t < L-1]            (through the predicted side)
//                 - w_al alpha^2 s_{t-1} p_t (1 - p_t) / N_AL [t > 0]      (through the LeftShift target:
//                                                   d BCE / d q = -logit(p_{t-1}) = -alpha s_{t-1})
//                 + w_cs alpha p_t (1 - p_t) prod_{t' != t} (1 - p_{c,t',i}) / N_CS
//   dJ/dWr[k,i] = sum_{c,t} x_{c,t,k} dJ/ds_{c,t,i};  dJ/db_i = sum_{c,t} dJ/ds_{c,t,i};
//   dJ/dx_{c,t,k} = sum_i dJ/ds_{c,t,i} Wr[k,i].
namespace {
double log_sigmoid(double z) { return z >= 0.0 ? -std::log1p(std::exp(-z)) : z - std::log1p(std::exp(z)); }
}  // namespace

extern "C" {

// x bf16 bits [C*L, d]; Wr [d, E]; br [E] or null.  Out: loss[2] = {L_AL, L_CS} (the unweighted objectives),
// dS [C*L, E], dWr [d, E], db [E] (may be null), dx [C*L, d] (may be null), all for J = w_al L_AL + w_cs L_CS.
int oracle_cls_losses(const uint16_t* x, int C, int L, int d, const float* Wr, const float* br, int E,
                      double alpha, double w_al, double w_cs, double* loss, double* dS, double* dWr, double* db,
                      double* dx) {
  if (C < 1 || L < 1 || d < 1 || E < 1) return 1;
  const int T = C * L;
  std::vector<double> s(static_cast<size_t>(T) * E), p(s.size());
  for (int t = 0; t < T; ++t)
    for (int i = 0; i < E; ++i) {
      double acc = 0.0;
      for (int k = 0; k < d; ++k)
        acc += widen_bf16(x[static_cast<size_t>(t) * d + k]) * static_cast<double>(Wr[static_cast<size_t>(k) * E + i]);
      if (br) acc += static_cast<double>(br[i]);
      s[static_cast<size_t>(t) * E + i] = acc;
      p[static_cast<size_t>(t) * E + i] = 1.0 / (1.0 + std::exp(-alpha * acc));
    }
  const double n_al = static_cast<double>(C) * (L - 1) * E, n_cs = static_cast<double>(C) * E;
  double l_al = 0.0, l_cs = 0.0;
  for (size_t q = 0; q < s.size(); ++q) dS[q] = 0.0;
  for (int c = 0; c < C; ++c)
    for (int i = 0; i < E; ++i) {
      double keep_all = 1.0;  // prod_t (1 - p)
      for (int t = 0; t < L; ++t) {
        const size_t q = (static_cast<size_t>(c) * L + t) * E + i;
        keep_all *= 1.0 - p[q];
        if (t + 1 < L) {
          // planted 11: the shift taken the other way (token t+1 predicts token t's pattern)
          const size_t pred = (g_mutation == 11) ? q + E : q, targ = (g_mutation == 11) ? q : q + E;
          const double y = p[targ];  // the next token's pattern
          const double z = alpha * s[pred];
          l_al += -(y * log_sigmoid(z) + (1.0 - y) * log_sigmoid(-z));
          dS[pred] += w_al * alpha * (p[pred] - y) / n_al;
          if (g_mutation != 9)  // planted 9: no gradient through the shifted target
            dS[targ] += -w_al * alpha * z * y * (1.0 - y) / n_al;
        }
      }
      l_cs += 1.0 - keep_all;
      for (int t = 0; t < L; ++t) {
        const size_t q = (static_cast<size_t>(c) * L + t) * E + i;
        double others = 1.0;  // prod_{t' != t} (1 - p)
        for (int u = 0; u < L; ++u)
          if (u != t || g_mutation == 10) others *= 1.0 - p[(static_cast<size_t>(c) * L + u) * E + i];  // planted 10
        dS[q] += w_cs * alpha * p[q] * (1.0 - p[q]) * others / n_cs;
      }
    }
  loss[0] = L > 1 ? l_al / n_al : 0.0;
  loss[1] = l_cs / n_cs;
  // dWr[k,i] = sum over t in ascending order (the loops run t outermost only to read x row by row)
  for (size_t q = 0; q < static_cast<size_t>(d) * E; ++q) dWr[q] = 0.0;
  for (int t = 0; t < T; ++t)
    for (int k = 0; k < d; ++k) {
      const double xv = widen_bf16(x[static_cast<size_t>(t) * d + k]);
      for (int i = 0; i < E; ++i) dWr[static_cast<size_t>(k) * E + i] += xv * dS[static_cast<size_t>(t) * E + i];
    }
  if (db)
    for (int i = 0; i < E; ++i) {
      double acc = 0.0;
      for (int t = 0; t < T; ++t) acc += dS[static_cast<size_t>(t) * E + i];
      db[i] = acc;
    }
  if (dx)
    for (int t = 0; t < T; ++t)
      for (int k = 0; k < d; ++k) {
        double acc = 0.0;
        for (int i = 0; i < E; ++i) acc += dS[static_cast<size_t>(t) * E + i] * static_cast<double>(Wr[static_cast<size_t>(k) * E + i]);
        dx[static_cast<size_t>(t) * d + k] = acc;
      }
  return 0;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------------
// Low-bit expert weights (the survey's low-bit quantisation of MoE weights, intelliparadigm survey, section
// 4.1; not a BlockFFN claim).  The format this build reads:
//   W1[e][j][k] = s1[e][j] * q1[e][j][k]          one power-of-two scale per row of W1 (over d)
//   W2[e][k][j] = t2[l] * s2[e][j] * q2[e][k][j]  one power-of-two scale per column of W2 (over d), written
//                                                  as a per-layer power of two t2 times a ratio s2 <= 1
// with q an fp8 e4m3 code (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no infinity; the
// largest finite value 448).  The scale of a row (column) is the smallest 2^m with 448 * 2^m >= its largest
// |w|; the code is w / 2^m rounded to the nearest e4m3 value, ties to the even code.  Every dequantised
// weight is then exactly a bf16 value.
namespace {
double e4m3_value(uint8_t code) {  // the value an e4m3 code stands for (NaN codes are never produced)
  const int sgn = code >> 7, ex = (code >> 3) & 15, man = code & 7;
  const double mag = ex == 0 ? std::ldexp(double(man), -9) : std::ldexp(1.0 + man / 8.0, ex - 7);
  return sgn ? -mag : mag;
}
// nearest e4m3 code to v (|v| <= 448), ties to the even code; the sign is kept (-0 for a negative input
// that rounds to zero).  The non-negative finite codes 0 .. 126 have increasing values, so the nearest is
// one of the two codes around |v|, found by bisection.
uint8_t e4m3_nearest(double v) {
  static const std::vector<double> values = [] {
    std::vector<double> t(127);
    for (int c = 0; c < 127; ++c) t[c] = e4m3_value(uint8_t(c));  // 0x7F is NaN
    return t;
  }();
  const uint8_t sgn = (std::signbit(v) ? 0x80 : 0x00);
  const double a = std::fabs(v);
  int lo = 0, hi = 126;  // values[lo] <= a < values[hi], or a at an end
  if (a >= values[126]) {
    lo = hi = 126;
  } else {
    while (hi - lo > 1) {
      const int mid = (lo + hi) / 2;
      if (values[mid] <= a) lo = mid;
      else hi = mid;
    }
  }
  const double dlo = a - values[lo], dhi = values[hi] - a;
  int best = (dlo < dhi || (dlo == dhi && (lo & 1) == 0)) ? lo : hi;
  if (g_mutation == 12) best = best > 0 ? best - 1 : 0;  // planted: rounds one code toward zero
  return uint8_t(sgn | best);
}
int pow2_exponent_for(double amax) {  // the smallest m with 448 * 2^m >= amax (0 for amax == 0)
  if (amax == 0.0) return 0;
  int m = -200;
  while (448.0 * std::ldexp(1.0, m) < amax) ++m;
  if (g_mutation == 13) ++m;  // planted: a scale twice too large
  return m;
}
}  // namespace

extern "C" {

double oracle_e4m3_value(int code) { return e4m3_value(uint8_t(code)); }
int oracle_e4m3_nearest(double v) { return e4m3_nearest(v); }

// W1 bf16 bits [NE, de, d], W2 bf16 bits [NE, d, de] for NE = n_layers * E experts (layer l owns experts
// l E .. l E + E - 1).  Out: q1 [NE, de, d], q2 [NE, d, de] codes, s1 [NE, de], s2 [NE, de], t2 [n_layers].
int oracle_quantize_fp8(const uint16_t* W1, const uint16_t* W2, int n_layers, int E, int d, int de, uint8_t* q1,
                        uint8_t* q2, float* s1, float* s2, float* t2) {
  if (n_layers < 1 || E < 1 || d < 1 || de < 1) return 1;
  const int NE = n_layers * E;
  std::vector<int> m2(static_cast<size_t>(NE) * de);
  for (int e = 0; e < NE; ++e)
    for (int j = 0; j < de; ++j) {
      const uint16_t* row = W1 + (static_cast<size_t>(e) * de + j) * d;
      double amax = 0.0;
      for (int k = 0; k < d; ++k) amax = std::max(amax, std::fabs(widen_bf16(row[k])));
      const int m = pow2_exponent_for(amax);
      s1[static_cast<size_t>(e) * de + j] = static_cast<float>(std::ldexp(1.0, m));
      for (int k = 0; k < d; ++k)
        q1[(static_cast<size_t>(e) * de + j) * d + k] = e4m3_nearest(std::ldexp(widen_bf16(row[k]), -m));
      double cmax = 0.0;
      for (int k = 0; k < d; ++k)
        cmax = std::max(cmax, std::fabs(widen_bf16(W2[(static_cast<size_t>(e) * d + k) * de + j])));
      m2[static_cast<size_t>(e) * de + j] = pow2_exponent_for(cmax);
    }
  for (int l = 0; l < n_layers; ++l) {
    int M = -100000;
    for (int e = l * E; e < (l + 1) * E; ++e)
      for (int j = 0; j < de; ++j) M = std::max(M, m2[static_cast<size_t>(e) * de + j]);
    t2[l] = static_cast<float>(std::ldexp(1.0, M));
    for (int e = l * E; e < (l + 1) * E; ++e)
      for (int j = 0; j < de; ++j) {
        const int m = m2[static_cast<size_t>(e) * de + j];
        s2[static_cast<size_t>(e) * de + j] = static_cast<float>(std::ldexp(1.0, m - M));
        for (int k = 0; k < d; ++k) {
          const size_t q = (static_cast<size_t>(e) * d + k) * de + j;
          q2[q] = e4m3_nearest(std::ldexp(widen_bf16(W2[q]), -m));
        }
      }
  }
  return 0;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------------
// The layer's backward (the training side of the same layer, lsdiaocha.cn BlockFFN article, section 2; the
// pages print no backward, so it is the chain rule through the forward above, RMSNorm router only).  For
// upstream gradient dy [T, d] of y:
//   q_{t,e} = W2_e^T dy_t                       (de)
//   dr_{t,e} = h_{t,e} . q_{t,e},  h = Swish(u), u = W1_e x_t
//   du_{t,e} = r_{t,e} q_{t,e} * Swish'(u),  Swish'(u) = sig(u) (1 + u (1 - sig(u)))
//   dW2_e += r_{t,e} dy_t h_{t,e}^T,  dW1_e += du_{t,e} x_t^T,  dx_t += W1_e^T du_{t,e}
//   r_i = g_i a_i / rho, a = relu(s), rho = sqrt(mean_i a_i^2):
//   dg_i += dr_i a_i / rho;  da_j = g_j dr_j / rho - a_j sum_i(dr_i g_i a_i) / (E rho^3);  ds = da [s > 0]
//   dWr += x_t ds_t^T,  db += ds_t,  dx_t += Wr ds_t
// A token with no positive s has r = 0 for every expert and gets no router gradient.  Every expert is
// evaluated (dense); an inactive one contributes exact zeros through r = 0.  Weights and x are fp64 here
// (the caller widens bf16), so finite differences can perturb any of them.
extern "C" {

// x [T,d], Wr [d,E], br [E] or null, g [E], W1 [E,de,d], W2 [E,d,de], dy [T,d]: all fp64.  Out (fp64): y
// [T,d] (the forward, for finite differences of J = sum dy . y), dx [T,d], dWr [d,E], db [E], dg [E],
// dW1 [E,de,d], dW2 [E,d,de].
int oracle_layer_backward(const double* x, int T, int d, const double* Wr, const double* br, const double* g,
                          const double* W1, const double* W2, int E, int de, const double* dy, double* y,
                          double* dx, double* dWr, double* db, double* dg, double* dW1, double* dW2) {
  if (T < 1 || d < 1 || E < 1 || de < 1) return 1;
  for (size_t q = 0; q < static_cast<size_t>(T) * d; ++q) y[q] = dx[q] = 0.0;
  for (size_t q = 0; q < static_cast<size_t>(d) * E; ++q) dWr[q] = 0.0;
  for (int i = 0; i < E; ++i) db[i] = dg[i] = 0.0;
  for (size_t q = 0; q < static_cast<size_t>(E) * de * d; ++q) dW1[q] = dW2[q] = 0.0;
  std::vector<double> s(E), a(E), r(E), dr(E), u(de), h(de), q(de);
  for (int t = 0; t < T; ++t) {
    const double* xt = x + static_cast<size_t>(t) * d;
    const double* dyt = dy + static_cast<size_t>(t) * d;
    double sumsq = 0.0;
    for (int i = 0; i < E; ++i) {
      double acc = br ? br[i] : 0.0;
      for (int k = 0; k < d; ++k) acc += xt[k] * Wr[static_cast<size_t>(k) * E + i];
      s[i] = acc;
      a[i] = acc > 0.0 ? acc : 0.0;
      sumsq += a[i] * a[i];
    }
    const double rho = std::sqrt(sumsq / E);
    for (int i = 0; i < E; ++i) r[i] = rho > 0.0 ? g[i] * a[i] / rho : 0.0;
    for (int e = 0; e < E; ++e) {
      const double* W1e = W1 + static_cast<size_t>(e) * de * d;
      const double* W2e = W2 + static_cast<size_t>(e) * d * de;
      for (int j = 0; j < de; ++j) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k) acc += W1e[static_cast<size_t>(j) * d + k] * xt[k];
        u[j] = acc;
        h[j] = acc / (1.0 + std::exp(-acc));
      }
      for (int k = 0; k < d; ++k) {
        double acc = 0.0;
        for (int j = 0; j < de; ++j) acc += W2e[static_cast<size_t>(k) * de + j] * h[j];
        y[static_cast<size_t>(t) * d + k] += r[e] * acc;
      }
      for (int j = 0; j < de; ++j) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k) acc += W2e[static_cast<size_t>(k) * de + j] * dyt[k];
        q[j] = acc;
      }
      double dre = 0.0;
      for (int j = 0; j < de; ++j) dre += h[j] * q[j];
      dr[e] = dre;
      for (int k = 0; k < d; ++k)
        for (int j = 0; j < de; ++j) dW2[(static_cast<size_t>(e) * d + k) * de + j] += r[e] * dyt[k] * h[j];
      for (int j = 0; j < de; ++j) {
        const double sg = 1.0 / (1.0 + std::exp(-u[j]));
        const double du = r[e] * q[j] * (g_mutation == 14 ? sg : sg * (1.0 + u[j] * (1.0 - sg)));  // planted 14
        for (int k = 0; k < d; ++k) {
          dW1[(static_cast<size_t>(e) * de + j) * d + k] += du * xt[k];
          dx[static_cast<size_t>(t) * d + k] += W1e[static_cast<size_t>(j) * d + k] * du;
        }
      }
    }
    if (rho > 0.0) {
      double c = 0.0;  // sum_i dr_i g_i a_i
      for (int i = 0; i < E; ++i) c += dr[i] * g[i] * a[i];
      for (int i = 0; i < E; ++i) {
        dg[i] += dr[i] * a[i] / rho;
        const double da = g[i] * dr[i] / rho - (g_mutation == 15 ? 0.0 : a[i] * c / (E * rho * rho * rho));  // planted 15
        const double ds = s[i] > 0.0 ? da : 0.0;
        db[i] += ds;
        for (int k = 0; k < d; ++k) {
          dWr[static_cast<size_t>(k) * E + i] += xt[k] * ds;
          dx[static_cast<size_t>(t) * d + k] += Wr[static_cast<size_t>(k) * E + i] * ds;
        }
      }
    }
  }
  return 0;
}

}  // extern "C"
