// QSA oracle: a plain, slow, host-only restatement of the Qwen Sparse Attention (QSA) layer.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file; only
// the tests, the smoke check and the benchmark's CPU-baseline leg do.  It shares no code, header,
// table or helper with the CUDA library.
//
// Source of the method: "Qwen3.8-Flash-Next architecture" (flozi.net), section "Der Weg eines
// Tokens durch das Modell", item 2 "Die zwei Stufen von QSA":
//   * the indexer projects tokens to light keys and averages groups of four keys into micro-block
//     keys                                                         -> pool_block_keys
//   * RoPE is applied after pooling                                 -> rope_pair / pool_block_keys
//   * blocks are scored with four query heads and one shared key head  -> index_scores_row
//   * per query the budget is 512 fully selected blocks (= 2048 tokens) plus the possibly
//     incomplete last block                                         -> select_topk_row, attend_row
//   * attention then runs over only the selected tokens (GQA)       -> attend_row
// and "Qwen3.8-Flash-Next" (studioglobal.ai), section "Hybride Aufmerksamkeit fuer sehr lange
// Kontexte": a compact index picks the relevant micro-blocks instead of attending everywhere.
//
// Readings where the pages are silent (each is listed with its reason in the design notes):
//   - head combination: s(t,b) = sum_h w_h * max(0, qi[t,h] . kp[b]) (LINEAR mode drops the max);
//   - candidates of query t are the complete blocks strictly before its own block, b < floor(t/blk);
//     the own block (tokens blk*floor(t/blk) .. t) is always attended and never scored;
//   - ties in the selection go to the lower block index; the selection is the top-k of the fp32
//     score (the precision the score is kept in), emitted in ascending block order, -1 padded;
//   - pooled keys and RoPE'd indexer vectors are stored as bf16 (round to nearest even);
//   - RoPE: half-split (NeoX) rotation, pair (i, i+Di/2), angle pos * theta^(-2i/Di); a pooled key
//     sits at the position of its block's first token;
//   - softmax scale is a parameter (1/sqrt(D) by default in the callers).
//
// Arithmetic: bf16 inputs are widened exactly; every sum, dot product, exponential and division is
// done in double.  Scores are rounded once to fp32; outputs once to bf16.
//
// Parity status of each function (pins live in tests/test_oracle_pins.py):
//   bf16_from_double, pool_block_keys, rope_pair, index_scores_row, select_topk_row, attend_row,
//   decode: pinned (closed forms, brute force, invariants, library routines).  Agreement with
//   numbers printed by the pages: parity unpinned -- the pages print no worked example; the only
//   printed check is 512 blocks x 4 tokens = 2048 tokens, which tests/golden/ pins.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

// QO_MUTANT != 0 builds a deliberately wrong oracle (one planted mistake per value) for the test
// that checks the pins catch such mistakes; the default build is QO_MUTANT == 0.
#ifndef QO_MUTANT
#define QO_MUTANT 0
#endif

namespace {

// ---- bf16 <-> double, from the IEEE-754 binary16-brain layout (1 sign, 8 exponent, 7 fraction) ----

double bf16_to_double(uint16_t h) {
  uint32_t bits = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return static_cast<double>(f);
}

// Round a double to the nearest bf16 value, ties to even, in one rounding step.
uint16_t bf16_from_double(double x) {
  if (std::isnan(x)) return 0x7FC0;
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0x0000;
  double a = std::fabs(x);
  if (a == 0.0) return sign;
  if (std::isinf(a)) return sign | 0x7F80;
  int e = 0;
  std::frexp(a, &e);                       // a = m * 2^e, m in [0.5, 1)
  // bf16 keeps 8 significant bits for normals (exponent >= -126) and a fixed quantum 2^-133 below.
  int qexp = std::max(e - 8, -133);
  double units = std::ldexp(a, -qexp);     // exact: a scaled to integer quanta (plus a fraction)
  double fl = std::floor(units);
  double frac = units - fl;
  double r = fl;
  if (QO_MUTANT != 11 && (frac > 0.5 || (frac == 0.5 && std::fmod(fl, 2.0) != 0.0))) r = fl + 1.0;
  double v = std::ldexp(r, qexp);          // exactly representable in fp32 (or 2^128 -> inf)
  if (v >= 0x1p128) return sign | 0x7F80;
  float f = static_cast<float>(v);
  uint32_t bits;
  std::memcpy(&bits, &f, sizeof bits);
  return sign | static_cast<uint16_t>(bits >> 16);
}

// YaRN context extension of the rotary frequencies (B. Peng, J. Quesnelle, H. Fan, E. Shippole,
// "YaRN: Efficient Context Window Extension of Large Language Models", 2023, sections 3.2 and 3.4;
// the pages name YaRN for the 1M-token context but give no parameters, so they are the caller's).
// For a pair with base frequency f (radians per position) the wavelength is 2 pi / f and
// r = orig_ctx * f / (2 pi) is the number of rotations it makes over the original context.  With
// the ramp g = clamp((r - alpha) / (beta - alpha), 0, 1) the frequency becomes
//   f' = (1 - g) * f / factor + g * f
// (pairs that rotate fewer than alpha times are interpolated by the factor, those that rotate more
// than beta times keep their frequency), and the rotated pair is scaled by mscale (the paper's
// attention temperature, 0.1 ln(factor) + 1 unless given).  factor <= 1 is plain RoPE.
struct Yarn {
  double factor = 1.0, orig_ctx = 0.0, alpha = 1.0, beta = 32.0, mscale = 0.0;
};

double yarn_freq(double f, const Yarn& y) {
  if (y.factor <= 1.0) return f;
  const double kTwoPi = 6.283185307179586476925286766559;
  const double r = y.orig_ctx * f / kTwoPi;
  double g = (r - y.alpha) / (y.beta - y.alpha);
  g = std::min(1.0, std::max(0.0, g));
  if (QO_MUTANT == 12) g = 1.0 - g;
  return (1.0 - g) * f / y.factor + g * f;
}

double yarn_mscale(const Yarn& y) {
  if (y.factor <= 1.0) return 1.0;
  return y.mscale > 0.0 ? y.mscale : 0.1 * std::log(y.factor) + 1.0;
}

// Half-split rotation of one (x1, x2) pair at position pos with frequency index i of Di/2.
void rope_pair(double x1, double x2, double pos, int64_t i, int64_t Di, double theta,
               double* y1, double* y2, const Yarn& yarn = Yarn()) {
  double inv_freq = std::pow(theta, -2.0 * static_cast<double>(i) / static_cast<double>(Di));
  inv_freq = yarn_freq(inv_freq, yarn);
  double ang = pos * inv_freq;
  double c = std::cos(ang), s = std::sin(ang);
  const double m = yarn_mscale(yarn);
  *y1 = m * (QO_MUTANT == 7 ? x1 * c + x2 * s : x1 * c - x2 * s);
  *y2 = m * (x2 * c + x1 * s);
}

// One indexer score row: s[b] for b < nb, the candidates of the query whose (already rotated)
// indexer vectors are qi_row[Hi][Di].
void index_scores_row(const uint16_t* qi_row, const uint16_t* kp, const float* head_w,
                      int64_t Hi, int64_t Di, int64_t nb, int mode, float* s) {
  std::vector<double> q(static_cast<size_t>(Hi * Di));
  for (int64_t i = 0; i < Hi * Di; ++i) q[i] = bf16_to_double(qi_row[i]);
  std::vector<double> kb(static_cast<size_t>(Di));
  for (int64_t b = 0; b < nb; ++b) {
    for (int64_t d = 0; d < Di; ++d) kb[d] = bf16_to_double(kp[b * Di + d]);
    double acc = 0.0;
    for (int64_t h = 0; h < Hi; ++h) {
      double dot = 0.0;
      for (int64_t d = 0; d < Di; ++d) dot += (QO_MUTANT == 9 ? q[d * Hi + h] : q[h * Di + d]) * kb[d];
      double term = (mode == 0 && QO_MUTANT != 1) ? std::max(0.0, dot) : dot;
      double w = (head_w && QO_MUTANT != 14) ? static_cast<double>(head_w[h]) : 1.0;
      acc += w * term;
    }
    s[b] = static_cast<float>(acc);
  }
}

// Top-k of an fp32 score row: the k largest scores, equal scores to the lower index, emitted in
// ascending index order and padded with -1.  kth[0] = k-th largest score, kth[1] = (k+1)-th
// (-inf when it does not exist).  Returns the number of selected entries.
int64_t select_topk_row(const float* s, int64_t n, int64_t k, int32_t* idx, float* kth) {
  std::vector<int32_t> order(static_cast<size_t>(n));
  for (int64_t i = 0; i < n; ++i) order[i] = static_cast<int32_t>(i);
  std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
    if (s[a] != s[b]) return s[a] > s[b];
    return QO_MUTANT == 2 ? a > b : a < b;
  });
  int64_t m = std::min(n, k);
  std::vector<int32_t> chosen(order.begin(), order.begin() + m);
  std::sort(chosen.begin(), chosen.end());
  for (int64_t i = 0; i < k; ++i) idx[i] = i < m ? chosen[i] : -1;
  if (kth) {
    const float ninf = -std::numeric_limits<float>::infinity();
    kth[0] = (n >= k && k > 0) ? s[order[k - 1]] : ninf;
    kth[1] = (n > k) ? s[order[k]] : ninf;
  }
  return m;
}

// Exact softmax attention of one query over its selected token set
//   S(pos) = { blk*b + j : b in idx, j < blk }  U  { blk*floor(pos/blk) .. pos }.
// q_row [Hq][D]; kb, vb point at token 0 of a [L][Hkv][D] cache.  Query head h reads KV head
// h / (Hq/Hkv).  Entries -1 and entries equal to the own block are skipped.
// Returns 0, or -1 when an entry lies outside [0, floor(pos/blk)].
int attend_row(const uint16_t* q_row, const uint16_t* kb, const uint16_t* vb, int64_t pos,
               const int32_t* idx, int64_t k, int64_t Hq, int64_t Hkv, int64_t D, int64_t blk,
               double scale, uint16_t* out, float* lse) {
  const int64_t own = pos / blk;
  std::vector<int64_t> toks;
  toks.reserve(static_cast<size_t>(k * blk + blk));
  for (int64_t i = 0; i < k; ++i) {
    int64_t b = idx[i];
    if (b == -1 || b == own) continue;
    if (b < 0 || b > own) return -1;
    for (int64_t j = 0; j < blk; ++j) toks.push_back(b * blk + j);
  }
  for (int64_t j = own * blk; j <= pos - (QO_MUTANT == 4 ? 1 : 0); ++j) toks.push_back(j);
  const int64_t group = Hq / Hkv;
  const size_t n = toks.size();
  std::vector<double> z(n), q(static_cast<size_t>(D)), o(static_cast<size_t>(D));
  for (int64_t h = 0; h < Hq; ++h) {
    const int64_t g = QO_MUTANT == 5 ? h % Hkv : h / group;
    for (int64_t d = 0; d < D; ++d) q[d] = bf16_to_double(q_row[h * D + d]);
    double zmax = -INFINITY;
    for (size_t i = 0; i < n; ++i) {
      const uint16_t* kr = kb + (toks[i] * Hkv + g) * D;
      double dot = 0.0;
      for (int64_t d = 0; d < D; ++d) dot += q[d] * bf16_to_double(kr[d]);
      z[i] = QO_MUTANT == 8 ? dot : dot * scale;
      zmax = std::max(zmax, z[i]);
    }
    double l = 0.0;
    std::fill(o.begin(), o.end(), 0.0);
    for (size_t i = 0; i < n; ++i) {
      double p = std::exp(z[i] - zmax);
      l += p;
      const uint16_t* vr = vb + (toks[i] * Hkv + g) * D;
      for (int64_t d = 0; d < D; ++d) o[d] += p * bf16_to_double(vr[d]);
    }
    for (int64_t d = 0; d < D; ++d) out[h * D + d] = bf16_from_double(o[d] / l);
    if (lse) lse[h] = static_cast<float>(QO_MUTANT == 13 ? std::log(l) : zmax + std::log(l));
  }
  return 0;
}

int resolve_threads(int nthreads) {
  if (nthreads > 0) return nthreads;
  unsigned hc = std::thread::hardware_concurrency();
  return hc ? static_cast<int>(hc) : 1;
}

template <class F>
void parallel_rows(int64_t n, int nthreads, F&& f) {
  int nt = static_cast<int>(std::min<int64_t>(resolve_threads(nthreads), std::max<int64_t>(n, 1)));
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    for (;;) {
      int64_t i = next.fetch_add(1);
      if (i >= n) break;
      f(i);
    }
  };
  if (nt <= 1) { worker(); return; }
  std::vector<std::thread> pool;
  for (int i = 0; i < nt; ++i) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

int qo_version() { return 1; }

int qo_hardware_threads() { return resolve_threads(0); }

void qo_bf16_round_f64(const double* x, uint16_t* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = bf16_from_double(x[i]);
}

// ki [B][L][Di] -> kp [B][floor(L/blk)][Di]: the mean of each group of blk consecutive keys, then
// (theta > 0) the half-split rotation at position pos0 + blk*b, then bf16 rounding.
void qo_pool_block_keys_yarn(const uint16_t* ki, uint16_t* kp, int64_t B, int64_t L, int64_t Di,
                             int64_t blk, double rope_theta, int64_t pos0, double yarn_factor,
                             double yarn_orig_ctx, double yarn_alpha, double yarn_beta,
                             double yarn_mscale) {
  Yarn yarn;
  yarn.factor = yarn_factor;
  yarn.orig_ctx = yarn_orig_ctx;
  yarn.alpha = yarn_alpha;
  yarn.beta = yarn_beta;
  yarn.mscale = yarn_mscale;
  const int64_t nb = L / blk;
  std::vector<double> m(static_cast<size_t>(Di));
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t j = 0; j < nb; ++j) {
      for (int64_t d = 0; d < Di; ++d) {
        double acc = 0.0;
        for (int64_t t = 0; t < blk - (QO_MUTANT == 6 ? 1 : 0); ++t) acc += bf16_to_double(ki[(b * L + j * blk + t) * Di + d]);
        m[d] = acc / static_cast<double>(blk);
      }
      uint16_t* dst = kp + (b * nb + j) * Di;
      if (rope_theta > 0.0) {
        const double pos = static_cast<double>(pos0 + j * blk + (QO_MUTANT == 10 ? blk - 1 : 0));
        for (int64_t i = 0; i < Di / 2; ++i) {
          double y1, y2;
          rope_pair(m[i], m[i + Di / 2], pos, i, Di, rope_theta, &y1, &y2, yarn);
          dst[i] = bf16_from_double(y1);
          dst[i + Di / 2] = bf16_from_double(y2);
        }
      } else {
        for (int64_t d = 0; d < Di; ++d) dst[d] = bf16_from_double(m[d]);
      }
    }
  }
}

void qo_pool_block_keys(const uint16_t* ki, uint16_t* kp, int64_t B, int64_t L, int64_t Di,
                        int64_t blk, double rope_theta, int64_t pos0) {
  qo_pool_block_keys_yarn(ki, kp, B, L, Di, blk, rope_theta, pos0, 1.0, 0.0, 1.0, 32.0, 0.0);
}

// Rotate rows of indexer queries x [rows][H][Di] at positions pos[rows] (YaRN-scaled when
// yarn_factor > 1); bf16 out.
void qo_rope_rows_yarn(const uint16_t* x, uint16_t* y, int64_t rows, int64_t H, int64_t Di,
                       const int64_t* pos, double theta, double yarn_factor, double yarn_orig_ctx,
                       double yarn_alpha, double yarn_beta, double yarn_mscale) {
  Yarn yarn;
  yarn.factor = yarn_factor;
  yarn.orig_ctx = yarn_orig_ctx;
  yarn.alpha = yarn_alpha;
  yarn.beta = yarn_beta;
  yarn.mscale = yarn_mscale;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t h = 0; h < H; ++h) {
      const uint16_t* src = x + (r * H + h) * Di;
      uint16_t* dst = y + (r * H + h) * Di;
      for (int64_t i = 0; i < Di / 2; ++i) {
        double y1, y2;
        rope_pair(bf16_to_double(src[i]), bf16_to_double(src[i + Di / 2]),
                  static_cast<double>(pos[r]), i, Di, theta, &y1, &y2, yarn);
        dst[i] = bf16_from_double(y1);
        dst[i + Di / 2] = bf16_from_double(y2);
      }
    }
  }
}

void qo_rope_rows(const uint16_t* x, uint16_t* y, int64_t rows, int64_t H, int64_t Di,
                  const int64_t* pos, double theta) {
  qo_rope_rows_yarn(x, y, rows, H, Di, pos, theta, 1.0, 0.0, 1.0, 32.0, 0.0);
}

void qo_index_scores(const uint16_t* qi_row, const uint16_t* kp, const float* head_w, int64_t Hi,
                     int64_t Di, int64_t nb, int mode, float* s) {
  index_scores_row(qi_row, kp, head_w, Hi, Di, nb, mode, s);
}

int64_t qo_select_topk(const float* s, int64_t n, int64_t k, int32_t* idx, float* kth) {
  return select_topk_row(s, n, k, idx, kth);
}

int qo_attend(const uint16_t* q_row, const uint16_t* kb, const uint16_t* vb, int64_t pos,
              const int32_t* idx, int64_t k, int64_t Hq, int64_t Hkv, int64_t D, int64_t blk,
              double scale, uint16_t* out, float* lse) {
  return attend_row(q_row, kb, vb, pos, idx, k, Hq, Hkv, D, blk, scale, out, lse);
}

// The whole layer for selected query rows of a prefill.
//   q  [B][Tq][Hq][D], k/v [B][Tk][Hkv][D], qi [B][Tq][Hi][Di] (not rotated), kp [B][NBk][Di]
//   (pooled and, if theta > 0, rotated by qo_pool_block_keys); query row t of batch b sits at
//   position q_pos0 + t.  rows = n_rows pairs (b, t).
//   idx_in == NULL: select with the indexer (scores, top-k), write idx_out [n_rows][k] and
//   kth [n_rows][2].  idx_in != NULL: attend over the given idx_in [n_rows][k].
//   out [n_rows][Hq][D] bf16, lse [n_rows][Hq] (natural log, scaled logits).
// Returns 0, or -1 when some row had an index outside its causal range.
int qo_prefill_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* qi,
                    const uint16_t* kp, const float* head_w, int64_t B, int64_t Tq, int64_t Tk,
                    int64_t NBk, int64_t Hq, int64_t Hkv, int64_t D, int64_t Hi, int64_t Di,
                    int64_t blk, int64_t topk, int64_t q_pos0, double rope_theta, int mode,
                    double scale, const int64_t* rows, int64_t n_rows, const int32_t* idx_in,
                    int32_t* idx_out, float* kth, uint16_t* out, float* lse, int nthreads) {
  (void)B;
  std::atomic<int> bad{0};
  parallel_rows(n_rows, nthreads, [&](int64_t r) {
    const int64_t b = rows[2 * r], t = rows[2 * r + 1];
    const int64_t pos = q_pos0 + t;
    const int32_t* idx = nullptr;
    std::vector<int32_t> sel;
    if (idx_in) {
      idx = idx_in + r * topk;
    } else {
      std::vector<uint16_t> qrow(static_cast<size_t>(Hi * Di));
      const uint16_t* src = qi + (b * Tq + t) * Hi * Di;
      if (rope_theta > 0.0) {
        qo_rope_rows(src, qrow.data(), 1, Hi, Di, &pos, rope_theta);
      } else {
        std::memcpy(qrow.data(), src, sizeof(uint16_t) * Hi * Di);
      }
      const int64_t nb = std::min(pos / blk + (QO_MUTANT == 3 ? 1 : 0), NBk);
      std::vector<float> s(static_cast<size_t>(std::max<int64_t>(nb, 1)));
      index_scores_row(qrow.data(), kp + (QO_MUTANT == 15 ? 0 : b) * NBk * Di, head_w, Hi, Di, nb, mode, s.data());
      sel.assign(static_cast<size_t>(topk), -1);
      select_topk_row(s.data(), nb, topk, sel.data(), kth ? kth + 2 * r : nullptr);
      if (idx_out) std::memcpy(idx_out + r * topk, sel.data(), sizeof(int32_t) * topk);
      idx = sel.data();
    }
    int rc = attend_row(q + (b * Tq + t) * Hq * D, k + b * Tk * Hkv * D, v + b * Tk * Hkv * D, pos,
                        idx, topk, Hq, Hkv, D, blk, scale, out + r * Hq * D,
                        lse ? lse + r * Hq : nullptr);
    if (rc) bad.store(1);
  });
  return bad.load() ? -1 : 0;
}

// One decode step for selected sequences: sequence b holds seqlen[b] tokens (the new token
// included) in caches k/v [B][Lmax][Hkv][D]; its query (q [B][Hq][D], qi [B][Hi][Di]) sits at
// position seqlen[b]-1; kp [B][NBk][Di] is the pooled indexer-key cache.
int qo_decode(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, const uint16_t* qi,
              const uint16_t* kp, const float* head_w, const int32_t* seqlens, int64_t B,
              int64_t Lmax, int64_t NBk, int64_t Hq, int64_t Hkv, int64_t D, int64_t Hi,
              int64_t Di, int64_t blk, int64_t topk, double rope_theta, int mode, double scale,
              const int64_t* seqs, int64_t n_seqs, const int32_t* idx_in, int32_t* idx_out,
              float* kth, uint16_t* out, float* lse, int nthreads) {
  (void)B;
  std::atomic<int> bad{0};
  parallel_rows(n_seqs, nthreads, [&](int64_t r) {
    const int64_t b = seqs[r];
    const int64_t pos = static_cast<int64_t>(seqlens[b]) - 1;
    const int32_t* idx = nullptr;
    std::vector<int32_t> sel;
    if (idx_in) {
      idx = idx_in + r * topk;
    } else {
      std::vector<uint16_t> qrow(static_cast<size_t>(Hi * Di));
      const uint16_t* src = qi + b * Hi * Di;
      if (rope_theta > 0.0) {
        qo_rope_rows(src, qrow.data(), 1, Hi, Di, &pos, rope_theta);
      } else {
        std::memcpy(qrow.data(), src, sizeof(uint16_t) * Hi * Di);
      }
      const int64_t nb = std::min(pos / blk + (QO_MUTANT == 3 ? 1 : 0), NBk);
      std::vector<float> s(static_cast<size_t>(std::max<int64_t>(nb, 1)));
      index_scores_row(qrow.data(), kp + (QO_MUTANT == 15 ? 0 : b) * NBk * Di, head_w, Hi, Di, nb, mode, s.data());
      sel.assign(static_cast<size_t>(topk), -1);
      select_topk_row(s.data(), nb, topk, sel.data(), kth ? kth + 2 * r : nullptr);
      if (idx_out) std::memcpy(idx_out + r * topk, sel.data(), sizeof(int32_t) * topk);
      idx = sel.data();
    }
    int rc = attend_row(q + b * Hq * D, kc + b * Lmax * Hkv * D, vc + b * Lmax * Hkv * D, pos, idx,
                        topk, Hq, Hkv, D, blk, scale, out + r * Hq * D,
                        lse ? lse + r * Hq : nullptr);
    if (rc) bad.store(1);
  });
  return bad.load() ? -1 : 0;
}

}  // extern "C"
