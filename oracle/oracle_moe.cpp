// oracle_moe.cpp -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, fp64 CPU restatement of the mixture-of-experts expert layer
// (router logits -> top-k + softmax -> grouping by expert -> dequantised int4
// gate/up/down projections with SwiGLU -> weighted combine).  It exists to
// check the CUDA library; only the tests, the smoke entry point and the
// benchmark's CPU-baseline leg may load it.  It shares no code, header, table
// or helper with the CUDA path.
//
// Sources (page title + section; the pages describe the method, not code):
//  * "两天移植，预填充提速8倍：Strata引擎实测" (kongchang.com), section
//    "Strata快在哪", MoE note: every layer holds many experts (512) and each
//    token activates only a few of them (10); bigger prefill batches mean each
//    expert is reused by more tokens (grouping tokens by expert).
//  * penglei.dev "Strata local MoE" post, section "原理一：把显存作为专家缓存":
//    the per-layer router selects a subset of experts for every token.
//  * lqnn.cn static review, section 3.1, and the yfxerp.com review, section
//    3.1: weights are group-quantised to 4 bit with per-group scales, group
//    size 32/64/128, scales computed per matrix.
//  * yfxerp.com review, section 5.1: the activation is fused with the FFN
//    projection; lqnn.cn review sections 1.2 and 6.2: dequantisation belongs
//    inside the matmul, never materialised beforehand (a GPU design point; the
//    oracle, being the definition, dequantises explicitly).
// The pages leave open the router formula, the tie-break, the activation and
// the combine; the readings used here are:
//  * logits l = x . W_r (+ b_e when a per-expert bias is given; the biased
//    logit is used both to select and to weight);
//  * top-k = the first k of a full stable sort by (logit desc, index asc);
//  * weights = softmax over the k selected logits;
//  * w = q * s exactly, q a two's-complement int4 in [-8, 7], low nibble =
//    even k, high nibble = odd k, s an fp16 scale per `group` elements of K;
//  * expert FFN = SwiGLU: h = SiLU(x.Wg) * (x.Wu), o = h.Wd, SiLU(z)=z/(1+e^-z);
//  * y_t = sum_j w_j o_j.
// Every function below is pinned by the CPU tests (brute force, closed forms,
// invariants); none is "parity unpinned".

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

namespace {

// bf16 bit pattern -> value: a bf16 is the top half of an IEEE-754 binary32.
double bf16_value(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// IEEE-754 binary16 bit pattern -> value (sign, 5-bit exponent with bias 15,
// 10-bit fraction; exponent 0 = subnormal; exponent 31 = inf/nan).
double f16_value(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int exponent = (h >> 10) & 0x1F;
  const int fraction = h & 0x3FF;
  double v;
  if (exponent == 0) {
    v = std::ldexp(static_cast<double>(fraction), -24);          // 2^-14 * f/1024
  } else if (exponent == 31) {
    v = fraction ? std::nan("") : INFINITY;
  } else {
    v = std::ldexp(1.0 + fraction / 1024.0, exponent - 15);
  }
  return sign ? -v : v;
}

// Signed value of nibble `kk` of a packed row: byte kk/2, low nibble for even
// kk, high nibble for odd kk, read as two's complement.
int int4_at(const uint8_t* row, int64_t kk) {
  const uint8_t byte = row[kk >> 1];
  const int nib = (kk & 1) ? (byte >> 4) : (byte & 0xF);
  return nib >= 8 ? nib - 16 : nib;
}

// Dequantised weight W[kk] of output feature row `nn`: q * s, exact in fp64.
double weight_at(const uint8_t* q, const uint16_t* s, int64_t K, int64_t G,
                 int64_t nn, int64_t kk) {
  const uint8_t* row = q + nn * (K / 2);
  const uint16_t* srow = s + nn * (K / G);
  return static_cast<double>(int4_at(row, kk)) * f16_value(srow[kk / G]);
}

// Dot product of an fp64 vector v[K] with dequantised row `nn`:
// sum_kk v[kk] * (q[nn][kk] * s[nn][kk/G]), visiting K group by group so each
// group's scale is decoded once.
double dot_row(const double* v, const uint8_t* q, const uint16_t* s, int64_t K,
               int64_t G, int64_t nn) {
  const uint8_t* row = q + nn * (K / 2);
  const uint16_t* srow = s + nn * (K / G);
  double acc = 0.0;
  for (int64_t g = 0; g < K / G; ++g) {
    const double scale = f16_value(srow[g]);
    for (int64_t kk = g * G; kk < (g + 1) * G; ++kk)
      acc += v[kk] * (static_cast<double>(int4_at(row, kk)) * scale);
  }
  return acc;
}

// Value of a 16-bit pattern stored as fp16 (is_f16 != 0) or bf16.
double half_value(uint16_t v, int is_f16) { return is_f16 ? f16_value(v) : bf16_value(v); }

}  // namespace

extern "C" {

// Exposed so the tests can pin the two scalar decoders against library
// conversions over every bit pattern.
double oracle_bf16_to_f64(uint16_t b) { return bf16_value(b); }
double oracle_f16_to_f64(uint16_t h) { return f16_value(h); }

// Dequantise rows [row0, row0+nrows) of one K-major packed matrix into
// out[nrows][K] (fp64).  q: [N][K/2] bytes, s: [N][K/G] fp16 bits.
void oracle_dequant_rows(const uint8_t* q, const uint16_t* s, int64_t N,
                         int64_t K, int64_t G, int64_t row0, int64_t nrows,
                         double* out) {
  (void)N;
  for (int64_t r = 0; r < nrows; ++r)
    for (int64_t kk = 0; kk < K; ++kk)
      out[r * K + kk] = weight_at(q, s, K, G, row0 + r, kk);
}

// Router logits (the router "selects experts per token"; formula is the plain
// linear router): logits[t][e] = sum_i x[t][i] * W_r[i][e] (+ bias[e]).
// x: [T][d] bf16 bits, w_router: [d][E] bf16 bits, bias: [E] fp32 or null.
void oracle_router_logits(const uint16_t* x, const uint16_t* w_router,
                          const float* bias, int64_t T, int64_t d, int64_t E,
                          double* logits) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int64_t i = 0; i < d; ++i)
        acc += bf16_value(x[t * d + i]) * bf16_value(w_router[i * E + e]);
      if (bias) acc += static_cast<double>(bias[e]);
      logits[t * E + e] = acc;
    }
  }
}

// Top-k selection and routing weights for each token: sort all E experts by
// (logit descending, expert index ascending) with a stable sort of the index
// list, keep the first k, then w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)
// over the k kept logits (l_0 the largest).  ids/w: [T][k] in that order.
void oracle_topk_softmax(const double* logits, int64_t T, int64_t E, int64_t k,
                         int32_t* ids, double* w) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const double* l = logits + t * E;
    std::vector<int32_t> order(E);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(),
                     [l](int32_t a, int32_t b) { return l[a] > l[b]; });
    double denom = 0.0;
    for (int64_t j = 0; j < k; ++j) denom += std::exp(l[order[j]] - l[order[0]]);
    for (int64_t j = 0; j < k; ++j) {
      ids[t * k + j] = order[j];
      w[t * k + j] = std::exp(l[order[j]] - l[order[0]]) / denom;
    }
  }
}

// Grouping by expert (the tokens that use one expert are processed together):
//   counts[e]  = number of slots s = t*k + j whose expert is e;
//   offsets    = exclusive prefix sum of counts, offsets[E] = T*k;
//   slot s with expert e goes to row offsets[e] + (number of earlier slots
//   s' < s with expert e); sorted_token[row] = s / k, slot_row[s] = row.
void oracle_permute(const int32_t* ids, int64_t T, int64_t k, int64_t E,
                    int32_t* counts, int32_t* offsets, int32_t* sorted_token,
                    int32_t* slot_row) {
  const int64_t S = T * k;
  for (int64_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t s = 0; s < S; ++s) counts[ids[s]] += 1;
  offsets[0] = 0;
  for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> filled(E, 0);
  for (int64_t s = 0; s < S; ++s) {
    const int32_t e = ids[s];
    const int32_t row = offsets[e] + filled[e]++;
    sorted_token[row] = static_cast<int32_t>(s / k);
    slot_row[s] = row;
  }
}

// One expert's SwiGLU FFN on one token row xt[d] (fp64):
//   g[j] = sum_i xt[i] Wg[e][j][i],  u[j] = sum_i xt[i] Wu[e][j][i],
//   h[j] = g[j] / (1 + exp(-g[j])) * u[j],  o[i'] = sum_j h[j] Wd[e][i'][j].
// Weights are K-major per output feature: gate/up [E][n][d/2], down [E][d][n/2].
// h_out[n] and o_out[d] receive the intermediate and the output.
void oracle_expert_ffn(const double* xt, const uint8_t* gate_q,
                       const uint16_t* gate_s, const uint8_t* up_q,
                       const uint16_t* up_s, const uint8_t* down_q,
                       const uint16_t* down_s, int64_t d, int64_t n, int64_t G,
                       int64_t e, double* h_out, double* o_out) {
  const uint8_t* gq = gate_q + e * n * (d / 2);
  const uint16_t* gs = gate_s + e * n * (d / G);
  const uint8_t* uq = up_q + e * n * (d / 2);
  const uint16_t* us = up_s + e * n * (d / G);
  const uint8_t* dq = down_q + e * d * (n / 2);
  const uint16_t* ds = down_s + e * d * (n / G);
  for (int64_t j = 0; j < n; ++j) {
    const double g = dot_row(xt, gq, gs, d, G, j);
    const double u = dot_row(xt, uq, us, d, G, j);
    h_out[j] = g / (1.0 + std::exp(-g)) * u;
  }
  for (int64_t i = 0; i < d; ++i) o_out[i] = dot_row(h_out, dq, ds, n, G, i);
}

// The whole layer for a subset of tokens (the oracle is per token, so a subset
// is exact).  Routing: logits from x and W_r (+bias), top-k + softmax as in
// oracle_topk_softmax, unless ids_in/w_in are given (then those routes are
// used as is: the tests feed the GPU's own routes to isolate the FFN).
//   tokens[n_sub]   token indices into x
//   y_out[n_sub][d] = sum_j w_j * o_j
//   ids_out/w_out   [n_sub][k] routes used (nullable)
//   h_out  [n_sub][k][n], o_out [n_sub][k][d] per-slot intermediates (nullable)
void oracle_moe_forward(const uint16_t* x, const uint16_t* w_router,
                        const float* bias, const uint8_t* gate_q,
                        const uint16_t* gate_s, const uint8_t* up_q,
                        const uint16_t* up_s, const uint8_t* down_q,
                        const uint16_t* down_s, int64_t T, int64_t d, int64_t E,
                        int64_t k, int64_t n, int64_t G, const int32_t* tokens,
                        int64_t n_sub, const int32_t* ids_in, const double* w_in,
                        double* y_out, int32_t* ids_out, double* w_out,
                        double* h_out, double* o_out) {
  (void)T;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n_sub; ++r) {
    const int64_t t = tokens[r];
    std::vector<double> xt(d), l(E), h(n), o(d), w(k);
    std::vector<int32_t> ids(k);
    for (int64_t i = 0; i < d; ++i) xt[i] = bf16_value(x[t * d + i]);
    if (ids_in) {
      for (int64_t j = 0; j < k; ++j) {
        ids[j] = ids_in[r * k + j];
        w[j] = w_in[r * k + j];
      }
    } else {
      oracle_router_logits(x + t * d, w_router, bias, 1, d, E, l.data());
      oracle_topk_softmax(l.data(), 1, E, k, ids.data(), w.data());
    }
    for (int64_t i = 0; i < d; ++i) y_out[r * d + i] = 0.0;
    for (int64_t j = 0; j < k; ++j) {
      oracle_expert_ffn(xt.data(), gate_q, gate_s, up_q, up_s, down_q, down_s,
                        d, n, G, ids[j], h.data(), o.data());
      for (int64_t i = 0; i < d; ++i) y_out[r * d + i] += w[j] * o[i];
      if (h_out) std::copy(h.begin(), h.end(), h_out + (r * k + j) * n);
      if (o_out) std::copy(o.begin(), o.end(), o_out + (r * k + j) * d);
    }
    if (ids_out) std::copy(ids.begin(), ids.end(), ids_out + r * k);
    if (w_out) std::copy(w.begin(), w.end(), w_out + r * k);
  }
}

// Weighted combine of given per-slot rows (fp64): y[t] = sum_j w[t][j] *
// rows[slot_row[t*k+j]].  rows are [S][d] fp16 (rows_f16 != 0) or bf16 bits.
void oracle_combine(const uint16_t* rows, int rows_f16, const double* w,
                    const int32_t* slot_row, int64_t T, int64_t k, int64_t d, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < k; ++j)
        acc += (w ? w[t * k + j] : 1.0) *
               half_value(rows[static_cast<int64_t>(slot_row[t * k + j]) * d + i], rows_f16);
      y[t * d + i] = acc;
    }
  }
}

// SwiGLU of one expert applied to given bf16 input rows (the gate/up
// projection alone): h[r][j] = SiLU(a_r . Wg[e][j]) * (a_r . Wu[e][j]).
// a: [R][d] bf16 bits, experts[R]: the expert of each row.  out: [R][n].
void oracle_gate_up_rows(const uint16_t* a, const int32_t* experts, int64_t R,
                         const uint8_t* gate_q, const uint16_t* gate_s,
                         const uint8_t* up_q, const uint16_t* up_s, int64_t d,
                         int64_t n, int64_t G, double* out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < R; ++r) {
    const int64_t e = experts[r];
    const uint8_t* gq = gate_q + e * n * (d / 2);
    const uint16_t* gs = gate_s + e * n * (d / G);
    const uint8_t* uq = up_q + e * n * (d / 2);
    const uint16_t* us = up_s + e * n * (d / G);
    std::vector<double> ar(d);
    for (int64_t i = 0; i < d; ++i) ar[i] = bf16_value(a[r * d + i]);
    for (int64_t j = 0; j < n; ++j) {
      const double g = dot_row(ar.data(), gq, gs, d, G, j);
      const double u = dot_row(ar.data(), uq, us, d, G, j);
      out[r * n + j] = g / (1.0 + std::exp(-g)) * u;
    }
  }
}

// The down projection alone on given rows: o[r][i] = a_r . Wd[e][i] (times
// scale[r] when given).  a: [R][n] fp16 (a_f16 != 0) or bf16 bits.  out: [R][d].
void oracle_down_rows(const uint16_t* a, int a_f16, const int32_t* experts, int64_t R,
                      const uint8_t* down_q, const uint16_t* down_s,
                      const float* scale, int64_t d, int64_t n, int64_t G,
                      double* out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < R; ++r) {
    const int64_t e = experts[r];
    const uint8_t* dq = down_q + e * d * (n / 2);
    const uint16_t* ds = down_s + e * d * (n / G);
    std::vector<double> ar(n);
    for (int64_t j = 0; j < n; ++j) ar[j] = half_value(a[r * n + j], a_f16);
    for (int64_t i = 0; i < d; ++i) {
      const double o = dot_row(ar.data(), dq, ds, n, G, i);
      out[r * d + i] = scale ? o * static_cast<double>(scale[r]) : o;
    }
  }
}

}  // extern "C"
