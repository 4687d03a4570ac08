// Plain, slow, CPU reference ("oracle") for one Qwen Sparse Attention layer
// with compression ratio 4 (QSA c4).  TEST INFRASTRUCTURE ONLY: the tests, the
// smoke check and the benchmark's CPU-baseline leg load it; the product path
// never does.  It shares no code with the CUDA path.
//
// Source of the method: the SGLang day-0 blog on Qwen3.8-Flash-Next, sections
// "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely" (indexer,
// compressed keys, top-512, expansion to at most 2051 positions, sparse GQA over
// raw K/V, 4-slot ring) and "IndexShare MTP: Reusing the QSA Selection Across
// Draft Steps" (frozen selection plus N+1 drafted positions).
//
// Precision: the blog fixes FP32 for the 4-key average; every other step runs
// in FP64.  Where the blog is silent or its text is garbled the readings below
// are used (each is listed with its reason in the design notes):
//   * score of block b:  s_b = sum_h w_h * max(0, q~_h . k^_b)      (formula lost in the text)
//   * ties in the top-512: the lower block index wins                 (unstated)
//   * "normalized" = divided by the L2 norm; a zero mean stays zero
//   * "rotated with the first token's MRoPE position": text-only positions make
//     the three MRoPE ids equal, i.e. plain RoPE; all 128 dims rotate, pairs
//     (i, i+64), inverse frequency theta^(-i/64), angles in FP64
//   * the rotated key and the rotated index query are each rounded once to
//     bf16 (round to nearest even), as stored / fed to a bf16 product
//   * only complete blocks (b < floor(L/4)) are scored; the L mod 4 newest
//     tokens are the tail that is always attended
//   * attention scale 1/sqrt(128); query head h reads KV head h / 8
//   * IndexShare draft query i (position L0+i) attends to the selection frozen
//     at position L0-1 plus positions L0 .. L0+i
//
// Layout of K and V here is logical, one request at a time: [token][kv_head][128].
// The paged layout is a storage detail of the GPU path and is not modelled.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

constexpr int D = 128;       // head dim of index heads and attention heads
constexpr int HI = 4;        // index query heads
constexpr int HQ = 16;       // attention query heads
constexpr int HKV = 2;       // attention KV heads
constexpr int C = 4;         // compression ratio
constexpr int TOPK = 512;    // kept blocks

double bf16_to_f64(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

float bf16_to_f32(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round an FP64 value to the nearest bf16 (ties to even), in one step.
// Written from the definition: bf16 keeps 8 significant bits and float's
// exponent range.  Handles zero, subnormal and overflow cases explicitly.
uint16_t f64_to_bf16(double x) {
  if (std::isnan(x)) return 0x7FC0;
  const bool neg = std::signbit(x);
  double a = std::fabs(x);
  uint16_t sign = neg ? 0x8000 : 0;
  if (a == 0.0) return sign;
  // quantum (ulp) of bf16 at |x|: 2^(e-7) for normal numbers, 2^-133 below 2^-126
  int e;
  std::frexp(a, &e);  // a = m * 2^e, m in [0.5, 1)  -> leading bit is 2^(e-1)
  int q = (e - 1) - 7;
  if (q < -133) q = -133;
  double scaled = std::ldexp(a, -q);  // exact: power-of-two scaling
  double fl = std::floor(scaled);
  double frac = scaled - fl;
  double r = fl;
  if (frac > 0.5 || (frac == 0.5 && std::fmod(fl, 2.0) != 0.0)) r = fl + 1.0;
  double y = std::ldexp(r, q);
  if (y >= 0x1.0p128) return sign | 0x7F80;  // rounds past the largest finite bf16
  float f = static_cast<float>(y);  // exact: y has <= 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(u >> 16) | sign;
}

// RoPE of one 128-vector at position pos (FP64 throughout).
void rope(const double* x, double pos, double theta, double* y) {
  for (int i = 0; i < D / 2; ++i) {
    const double inv_freq = std::pow(theta, -static_cast<double>(i) / (D / 2));
    const double ang = pos * inv_freq;
    const double c = std::cos(ang), s = std::sin(ang);
    y[i] = x[i] * c - x[i + D / 2] * s;
    y[i + D / 2] = x[i] * s + x[i + D / 2] * c;
  }
}

template <typename F>
void parallel(int64_t n, int nthreads, F&& f) {
  if (nthreads <= 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) f(i);
    return;
  }
  if (nthreads > n) nthreads = static_cast<int>(n);
  std::vector<std::thread> th;
  th.reserve(nthreads);
  for (int t = 0; t < nthreads; ++t)
    th.emplace_back([&, t] {
      for (int64_t i = t; i < n; i += nthreads) f(i);
    });
  for (auto& x : th) x.join();
}

}  // namespace

extern "C" {

int oracle_version() { return 1; }

// FP64 -> bf16 (exposed for the pins).
uint16_t oracle_f64_to_bf16(double x) { return f64_to_bf16(x); }

// RoPE of `nvec` 128-vectors given as FP64, each at its own position.
void oracle_rope_f64(const double* x, const double* pos, int64_t nvec, double theta, double* y) {
  for (int64_t v = 0; v < nvec; ++v) rope(x + v * D, pos[v], theta, y + v * D);
}

// One compressed index key from the 4 raw keys of block b (tokens 4b..4b+3):
// FP32 mean (summed in token order), L2-normalised and rotated at position 4b
// in FP64, rounded once to bf16.
void oracle_compress_block(const uint16_t* raw4, int64_t b, double theta, uint16_t* out) {
  float m[D];
  for (int d = 0; d < D; ++d) {
    float s = bf16_to_f32(raw4[d]);
    s = s + bf16_to_f32(raw4[D + d]);
    s = s + bf16_to_f32(raw4[2 * D + d]);
    s = s + bf16_to_f32(raw4[3 * D + d]);
    m[d] = s * 0.25f;
  }
  double n2 = 0.0;
  for (int d = 0; d < D; ++d) n2 += static_cast<double>(m[d]) * static_cast<double>(m[d]);
  const double n = std::sqrt(n2);
  double kh[D], kr[D];
  for (int d = 0; d < D; ++d) kh[d] = n > 0.0 ? static_cast<double>(m[d]) / n : 0.0;
  rope(kh, static_cast<double>(C * b), theta, kr);
  for (int d = 0; d < D; ++d) out[d] = f64_to_bf16(kr[d]);
}

// Compressed keys of a whole sequence: raw [n_tok][128] -> comp [n_tok/4][128].
void oracle_compress(const uint16_t* raw, int64_t n_tok, double theta, uint16_t* comp, int nthreads) {
  const int64_t nb = n_tok / C;
  parallel(nb, nthreads, [&](int64_t b) { oracle_compress_block(raw + b * C * D, b, theta, comp + b * D); });
}

// Token-by-token append with the 4-slot ring: the key of position `pos` goes to
// ring slot pos mod 4; the 4th key of a block completes it and its compressed
// key is written to comp[pos/4].
void oracle_append(uint16_t* ring, uint16_t* comp, const uint16_t* key, int64_t pos, double theta) {
  std::memcpy(ring + (pos % C) * D, key, D * sizeof(uint16_t));
  if (pos % C == C - 1) oracle_compress_block(ring, pos / C, theta, comp + (pos / C) * D);
}

// Index queries rotated at position pos and rounded to bf16: [nh][128] -> [nh][128].
void oracle_rotate_query(const uint16_t* q, int nh, int64_t pos, double theta, uint16_t* out) {
  double x[D], y[D];
  for (int h = 0; h < nh; ++h) {
    for (int d = 0; d < D; ++d) x[d] = bf16_to_f64(q[h * D + d]);
    rope(x, static_cast<double>(pos), theta, y);
    for (int d = 0; d < D; ++d) out[h * D + d] = f64_to_bf16(y[d]);
  }
}

// Block scores s_b = sum_h w_h * max(0, q~_h . k^_b) for b < nb, FP64.
void oracle_block_scores(const uint16_t* qrot, const float* w, const uint16_t* comp, int64_t nb, double* s) {
  double q[HI][D];
  for (int h = 0; h < HI; ++h)
    for (int d = 0; d < D; ++d) q[h][d] = bf16_to_f64(qrot[h * D + d]);
  for (int64_t b = 0; b < nb; ++b) {
    double k[D];
    for (int d = 0; d < D; ++d) k[d] = bf16_to_f64(comp[b * D + d]);
    double total = 0.0;
    for (int h = 0; h < HI; ++h) {
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += q[h][d] * k[d];
      total += static_cast<double>(w[h]) * std::max(0.0, dot);
    }
    s[b] = total;
  }
}

// Keep the best min(nb, k) blocks by (score descending, block index ascending);
// return their indices in ascending order.  Returns the count.
int32_t oracle_select_topk(const double* s, int64_t nb, int32_t k, int32_t* blocks) {
  if (nb <= k) {
    for (int64_t b = 0; b < nb; ++b) blocks[b] = static_cast<int32_t>(b);
    return static_cast<int32_t>(nb);
  }
  std::vector<int32_t> idx(nb);
  for (int64_t b = 0; b < nb; ++b) idx[b] = static_cast<int32_t>(b);
  std::sort(idx.begin(), idx.end(), [&](int32_t a, int32_t c) {
    if (s[a] != s[c]) return s[a] > s[c];
    return a < c;
  });
  idx.resize(k);
  std::sort(idx.begin(), idx.end());
  std::copy(idx.begin(), idx.end(), blocks);
  return k;
}

// Expansion: each kept block b -> positions 4b..4b+3, then the tail tokens
// 4*floor(L/4) .. L-1 of the unfinished block.  Returns the count (<= 2051).
int32_t oracle_expand(const int32_t* blocks, int32_t n, int64_t L, int32_t* pos) {
  int32_t m = 0;
  for (int32_t i = 0; i < n; ++i)
    for (int j = 0; j < C; ++j) pos[m++] = blocks[i] * C + j;
  for (int64_t p = (L / C) * C; p < L; ++p) pos[m++] = static_cast<int32_t>(p);
  return m;
}

// Sparse GQA of one query token over the given positions (FP64):
// head h uses KV head h/8; o_h = softmax_j(scale * q_h . K[pos_j]) V[pos_j].
// K, V: [token][2][128] bf16.  out: [16][128] FP64; lse: [16] (natural log), may be null.
void oracle_sparse_gqa(const uint16_t* q, const uint16_t* K, const uint16_t* V, const int32_t* pos, int32_t npos,
                       double scale, double* out, double* lse) {
  std::vector<double> logit(npos > 0 ? npos : 1);
  for (int h = 0; h < HQ; ++h) {
    const int g = h / (HQ / HKV);
    double qh[D];
    for (int d = 0; d < D; ++d) qh[d] = bf16_to_f64(q[h * D + d]);
    double mx = -INFINITY;
    for (int32_t j = 0; j < npos; ++j) {
      const uint16_t* kr = K + (static_cast<int64_t>(pos[j]) * HKV + g) * D;
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += qh[d] * bf16_to_f64(kr[d]);
      logit[j] = dot * scale;
      mx = std::max(mx, logit[j]);
    }
    double den = 0.0;
    double acc[D] = {0.0};
    for (int32_t j = 0; j < npos; ++j) {
      const double p = std::exp(logit[j] - mx);
      den += p;
      const uint16_t* vr = V + (static_cast<int64_t>(pos[j]) * HKV + g) * D;
      for (int d = 0; d < D; ++d) acc[d] += p * bf16_to_f64(vr[d]);
    }
    for (int d = 0; d < D; ++d) out[h * D + d] = npos > 0 ? acc[d] / den : 0.0;
    if (lse) lse[h] = npos > 0 ? mx + std::log(den) : -INFINITY;
  }
}

// E4M3 byte -> value, from the format's definition: sign bit, 4 exponent bits (bias 7), 3 mantissa
// bits; exponent 0 is subnormal (m/8 * 2^-6); exponent 15 with mantissa 7 is NaN (no infinities).
double e4m3_to_f64(uint8_t b) {
  const int sgn = b >> 7, e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e ? std::ldexp(1.0 + m / 8.0, e - 7) : std::ldexp(m / 8.0, -6);
  return sgn ? -mag : mag;
}

double oracle_e4m3_to_f64(uint8_t b) { return e4m3_to_f64(b); }

// Sparse GQA over FP8 K/V (reading: E4M3 codes with one scale for K and one for V, value = code *
// scale), FP64: head h uses KV head h/8; o_h = softmax_j(scale * q_h . K[pos_j]) V[pos_j].
// K8, V8: [token][2][128] E4M3 bytes.  out: [16][128] FP64; lse: [16] (natural log), may be null.
void oracle_sparse_gqa_fp8(const uint16_t* q, const uint8_t* K8, const uint8_t* V8, double k_scale, double v_scale,
                           const int32_t* pos, int32_t npos, double scale, double* out, double* lse) {
  std::vector<double> logit(npos > 0 ? npos : 1);
  for (int h = 0; h < HQ; ++h) {
    const int g = h / (HQ / HKV);
    double qh[D];
    for (int d = 0; d < D; ++d) qh[d] = bf16_to_f64(q[h * D + d]);
    double mx = -INFINITY;
    for (int32_t j = 0; j < npos; ++j) {
      const uint8_t* kr = K8 + (static_cast<int64_t>(pos[j]) * HKV + g) * D;
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += qh[d] * (e4m3_to_f64(kr[d]) * k_scale);
      logit[j] = dot * scale;
      mx = std::max(mx, logit[j]);
    }
    double den = 0.0;
    double acc[D] = {0.0};
    for (int32_t j = 0; j < npos; ++j) {
      const double p = std::exp(logit[j] - mx);
      den += p;
      const uint8_t* vr = V8 + (static_cast<int64_t>(pos[j]) * HKV + g) * D;
      for (int d = 0; d < D; ++d) acc[d] += p * (e4m3_to_f64(vr[d]) * v_scale);
    }
    for (int d = 0; d < D; ++d) out[h * D + d] = npos > 0 ? acc[d] / den : 0.0;
    if (lse) lse[h] = npos > 0 ? mx + std::log(den) : -INFINITY;
  }
}

// Selection of one query: rotate, score complete blocks, keep the top-512,
// expand with the tail.  comp must hold at least floor(L/4) blocks.
// Returns the number of positions; writes blocks (<=512), nblocks, pos (<=2051).
int32_t oracle_select_query(const uint16_t* idx_q, const float* w, const uint16_t* comp, int64_t L, double theta,
                            int32_t* blocks, int32_t* nblocks, int32_t* pos, double* scores_or_null) {
  uint16_t qrot[HI * D];
  oracle_rotate_query(idx_q, HI, L - 1, theta, qrot);
  const int64_t nb = L / C;
  std::vector<double> s(nb > 0 ? nb : 1);
  oracle_block_scores(qrot, w, comp, nb, s.data());
  if (scores_or_null) std::copy(s.begin(), s.begin() + nb, scores_or_null);
  const int32_t n = oracle_select_topk(s.data(), nb, TOPK, blocks);
  *nblocks = n;
  return oracle_expand(blocks, n, L, pos);
}

// One decode step for a batch of requests, each given by pointers to its own
// logical arrays.  Request r: context L[r] (including the new token at L[r]-1);
// ring[r] [4][128] and comp[r] [>= L/4][128] hold the state *before* the
// new key (they are updated in place, like the layer's cache); new_key[r] [128];
// idx_q[r] [4][128]; w[r] [4]; q[r] [16][128]; K[r], V[r] [>= L][2][128].
// Outputs: out[r] [16][128] FP64, blocks[r] [512], nblocks[r], pos[r] [2051], npos[r].
void oracle_decode_batch(int32_t B, const int64_t* L, uint16_t* const* ring, uint16_t* const* comp,
                         const uint16_t* const* new_key, const uint16_t* const* idx_q, const float* const* w,
                         const uint16_t* const* q, const uint16_t* const* K, const uint16_t* const* V, double theta,
                         double scale, double* const* out, int32_t* const* blocks, int32_t* nblocks,
                         int32_t* const* pos, int32_t* npos, int nthreads) {
  parallel(B, nthreads, [&](int64_t r) {
    oracle_append(ring[r], comp[r], new_key[r], L[r] - 1, theta);
    npos[r] = oracle_select_query(idx_q[r], w[r], comp[r], L[r], theta, blocks[r], &nblocks[r], pos[r], nullptr);
    oracle_sparse_gqa(q[r], K[r], V[r], pos[r], npos[r], scale, out[r], nullptr);
  });
}

// Prefill rows of one sequence: query t (position t, context t+1) for each t
// in `rows`.  comp: all compressed keys of the sequence.  idx_q [T][4][128],
// w [T][4], q [T][16][128] indexed by position.  Outputs per listed row i:
// out [i][16][128], blocks [i][512], nblocks[i], npos[i] (positions not kept).
void oracle_prefill_rows(const int64_t* rows, int64_t nrows, const uint16_t* idx_q, const float* w, const uint16_t* q,
                         const uint16_t* comp, const uint16_t* K, const uint16_t* V, double theta, double scale,
                         double* out, int32_t* blocks, int32_t* nblocks, int32_t* npos, int nthreads) {
  parallel(nrows, nthreads, [&](int64_t i) {
    const int64_t t = rows[i];
    std::vector<int32_t> p(TOPK * C + C);
    npos[i] = oracle_select_query(idx_q + t * HI * D, w + t * HI, comp, t + 1, theta, blocks + i * TOPK, &nblocks[i],
                                  p.data(), nullptr);
    if (out) oracle_sparse_gqa(q + t * HQ * D, K, V, p.data(), npos[i], scale, out + i * HQ * D, nullptr);
  });
}

// Index projection of n tokens (reading: the indexer's query heads, key and head weights are one
// bias-free linear map of the token's hidden state; the pages give neither the map nor the hidden
// size).  For token i and feature f: y = sum_j W[f][j] * x[i][j] in FP64.  Features 0..511 are the
// 4 index query heads (head h, dim d at 128h + d) and 512..639 the index key, each rounded once to
// bf16; 640..643 are the 4 head weights, rounded once to float.
// x: [n][hidden] bf16; W: [644][hidden] bf16; idx_q: [n][4][128]; idx_k: [n][128]; w: [n][4].
void oracle_index_project(const uint16_t* x, const uint16_t* W, int64_t n, int64_t hidden, uint16_t* idx_q,
                          uint16_t* idx_k, float* w, int nthreads) {
  constexpr int F = HI * D + D + HI;
  parallel(n, nthreads, [&](int64_t i) {
    const uint16_t* xi = x + i * hidden;
    for (int f = 0; f < F; ++f) {
      const uint16_t* wf = W + static_cast<int64_t>(f) * hidden;
      double y = 0.0;
      for (int64_t j = 0; j < hidden; ++j) y += bf16_to_f64(wf[j]) * bf16_to_f64(xi[j]);
      if (f < HI * D) {
        idx_q[i * HI * D + f] = f64_to_bf16(y);
      } else if (f < HI * D + D) {
        idx_k[i * D + (f - HI * D)] = f64_to_bf16(y);
      } else {
        w[i * HI + (f - HI * D - D)] = static_cast<float>(y);
      }
    }
  });
}

// IndexShare draft step of one request: draft query i (i = 0..n_plus_1-1) at
// position L0+i attends to the frozen positions (selected at position L0-1)
// plus positions L0..L0+i.  q: [n_plus_1][16][128]; out: [n_plus_1][16][128].
void oracle_indexshare(const int32_t* frozen, int32_t nfrozen, int64_t L0, int32_t n_plus_1, const uint16_t* q,
                       const uint16_t* K, const uint16_t* V, double scale, double* out) {
  std::vector<int32_t> p(nfrozen + n_plus_1);
  for (int i = 0; i < n_plus_1; ++i) {
    int32_t m = 0;
    for (int32_t j = 0; j < nfrozen; ++j) p[m++] = frozen[j];
    for (int64_t x = L0; x <= L0 + i; ++x) p[m++] = static_cast<int32_t>(x);
    oracle_sparse_gqa(q + i * HQ * D, K, V, p.data(), m, scale, out + i * HQ * D, nullptr);
  }
}

}  // extern "C"
