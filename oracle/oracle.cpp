// oracle.cpp -- plain, slow CPU oracle of one Llama-style decoder step.
//
// TEST INFRASTRUCTURE ONLY: loaded by tests/, __graft_entry__.smoke() and bench.py's
// cpu_baseline and reference arm, never by the product path.  Written from the pages
// alone; it shares no code with the CUDA library.
//
// The pages name the operations of a decode step but never write them out; this file
// takes the plainest reading (a standard Llama decoder), step by step:
//   x   = E[token]                                            (embedding)
//   per layer:
//     xn  = RMSNorm(x; g_attn)                                (Mirage, "Case 1: Normalization + Linear")
//     q,k,v = Wq xn, Wk xn, Wv xn                             (matmul, Mirage attention example)
//     q,k = LayerNorm per head (QK-norm models only)          (Mirage, "Case 4.1: Attention with
//                                                              Query-Key Normalization")
//     q,k = RoPE(q,k; pos)                                    (rotate-half pairing, reading below)
//     cache[pos] = k, v  (bf16-rounded when kv_round)         (KV-cache append)
//     o_h = sum_j softmax_j(q_h . k_j * scale) v_j,  j = 0..pos,  kv head of q head h = h*nkv/nq
//                                                             (Mirage attention example: O = softmax(QK)V)
//     x  += Wo o
//     xn  = RMSNorm(x; g_mlp)
//     x  += Wd (silu(Wg xn) * (Wu xn))                       (Mirage, "Case 3: Gated MLP")
//   logits = Wlm RMSNorm(x; g_final)
// Readings where the pages are silent:
//   * RMSNorm: y = x * (mean(x^2) + eps)^(-1/2) * g, the sum of squares in double.
//   * RoPE: pairs (i, i + d/2) of each head; angle = pos * theta^(-2i/d) in double; in the
//     fp32 mode cos and sin are rounded once to fp32 before use.
//   * QK-norm: a LayerNorm over the head_dim values of each query head and each key head,
//     with a gain and a bias per head and element, applied to the projections before RoPE
//     (so the cache holds normalised, rotated keys), eps = the model's rms_eps.
//   * scale = 1/sqrt(head_dim) in the decoder; the standalone op takes it as an argument
//     (1.0 for the Mirage example, which applies no scaling).
//   * GQA: contiguous groups, q head h reads kv head floor(h * nkv / nq).
//   * Accumulation: every dot product, norm and softmax sums in double; results are stored
//     in the activation type T (fp32, or fp64 in the f64 mode).  Dot products use four
//     interleaved partial sums (k mod 4), always in the same order, so results do not
//     depend on the thread count.
#include "oracle.h"

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <thread>
#include <vector>

namespace {

int g_threads = 0;

int threads() {
  if (g_threads > 0) return g_threads;
  const char* e = std::getenv("OR_THREADS");
  if (e && std::atoi(e) > 0) return std::atoi(e);
  unsigned n = std::thread::hardware_concurrency();
  return n ? (int)n : 1;
}

// Run f(lo, hi) over [0, n) split into contiguous blocks, one per worker.
template <class F>
void parallel_rows(int n, long long work_per_row, F f) {
  int nt = threads();
  if ((long long)n * work_per_row < (1LL << 18)) nt = 1;
  nt = std::max(1, std::min(nt, n));
  if (nt == 1) {
    f(0, n);
    return;
  }
  std::vector<std::thread> pool;
  int per = (n + nt - 1) / nt;
  for (int t = 0; t < nt; ++t) {
    int lo = t * per, hi = std::min(n, lo + per);
    if (lo >= hi) break;
    pool.emplace_back([=] { f(lo, hi); });
  }
  for (auto& th : pool) th.join();
}

inline double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

inline double f16_to_double(uint16_t h) {
  // IEEE binary16 -> double, exact
  int sign = (h >> 15) & 1, exp = (h >> 10) & 0x1f, man = h & 0x3ff;
  double v;
  if (exp == 0) v = std::ldexp((double)man, -24);
  else if (exp == 31) v = man ? NAN : INFINITY;
  else v = std::ldexp((double)(man | 0x400), exp - 25);
  return sign ? -v : v;
}

// Round a float to the nearest bf16 (ties to even) and return the bf16 bits.
inline uint16_t float_to_bf16_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)((u >> 16) | ((u & 0xffffu) ? 0x40u : 0u));
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

// Dot product of a bf16-widened weight row (already in double) with x, four fixed partial sums.
template <class T>
double dot_row(const double* w, const T* x, int n) {
  double s0 = 0, s1 = 0, s2 = 0, s3 = 0;
  int k = 0;
  for (; k + 4 <= n; k += 4) {
    s0 += w[k] * (double)x[k];
    s1 += w[k + 1] * (double)x[k + 1];
    s2 += w[k + 2] * (double)x[k + 2];
    s3 += w[k + 3] * (double)x[k + 3];
  }
  for (; k < n; ++k) s0 += w[k] * (double)x[k];
  return (s0 + s1) + (s2 + s3);
}

// Y[i][r] = sum_k W[r][k] X[i][k] for i < nvec; W bf16 [rows][cols]; X, Y in T.
template <class T>
void linear(const uint16_t* W, int rows, int cols, const T* X, int nvec, T* Y) {
  parallel_rows(rows, (long long)cols * nvec, [&](int lo, int hi) {
    std::vector<double> wrow(cols);
    for (int r = lo; r < hi; ++r) {
      const uint16_t* wr = W + (size_t)r * cols;
      for (int k = 0; k < cols; ++k) wrow[k] = bf16_to_double(wr[k]);
      for (int i = 0; i < nvec; ++i) Y[(size_t)i * rows + r] = (T)dot_row(wrow.data(), X + (size_t)i * cols, cols);
    }
  });
}

// RMSNorm (Mirage "Case 1"): y = x / sqrt(mean(x^2) + eps) * g.
template <class T>
void rmsnorm(const T* x, const uint16_t* g, int n, double eps, T* y) {
  double ss = 0;
  for (int i = 0; i < n; ++i) ss += (double)x[i] * (double)x[i];
  double r = 1.0 / std::sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) y[i] = (T)((double)x[i] * r * bf16_to_double(g[i]));
}

// LayerNorm (QK-norm, Mirage "Case 4.1"): y = (x - mean) / sqrt(var + eps) * g + b, the
// mean and the mean squared deviation in double.  In place is allowed (x == y).
template <class T>
void layernorm(const T* x, const uint16_t* g, const uint16_t* b, int n, double eps, T* y) {
  double sum = 0;
  for (int i = 0; i < n; ++i) sum += (double)x[i];
  const double mean = sum / n;
  double sq = 0;
  for (int i = 0; i < n; ++i) sq += ((double)x[i] - mean) * ((double)x[i] - mean);
  const double r = 1.0 / std::sqrt(sq / n + eps);
  for (int i = 0; i < n; ++i) y[i] = (T)(((double)x[i] - mean) * r * bf16_to_double(g[i]) + bf16_to_double(b[i]));
}

// Rotary angle table entry for pair i at position pos (reading: rotate-half, theta^(-2i/d)).
inline void rope_angle(int head_dim, int pos, double theta, int i, double* c, double* s) {
  double inv_freq = std::pow(theta, -2.0 * (double)i / (double)head_dim);
  double ang = (double)pos * inv_freq;
  *c = std::cos(ang);
  *s = std::sin(ang);
}

// Rotate one head vector in place: (v_i, v_{i+d/2}) -> (v_i c - v_{i+d/2} s, v_{i+d/2} c + v_i s).
template <class T>
void rope_head(T* v, int head_dim, int pos, double theta, bool round_table_to_f32) {
  int half = head_dim / 2;
  for (int i = 0; i < half; ++i) {
    double c, s;
    rope_angle(head_dim, pos, theta, i, &c, &s);
    if (round_table_to_f32) {
      c = (double)(float)c;
      s = (double)(float)s;
    }
    double a = (double)v[i], b = (double)v[i + half];
    v[i] = (T)(a * c - b * s);
    v[i + half] = (T)(b * c + a * s);
  }
}

// o = sum_j softmax_j(scale * q.k_j) v_j over L keys; k and v are [L][d], key-major.
template <class T, class KV>
void attend(const T* q, const KV* k, const KV* v, int L, int d, double scale, T* o, double* probs_out) {
  std::vector<double> s(L);
  double m = -INFINITY;
  for (int j = 0; j < L; ++j) {
    double acc = 0;
    for (int t = 0; t < d; ++t) acc += (double)q[t] * (double)k[(size_t)j * d + t];
    s[j] = acc * scale;
    m = std::max(m, s[j]);
  }
  double denom = 0;
  for (int j = 0; j < L; ++j) {
    s[j] = std::exp(s[j] - m);
    denom += s[j];
  }
  for (int t = 0; t < d; ++t) {
    double acc = 0;
    for (int j = 0; j < L; ++j) acc += s[j] * (double)v[(size_t)j * d + t];
    o[t] = (T)(acc / denom);
  }
  if (probs_out)
    for (int j = 0; j < L; ++j) probs_out[j] = s[j] / denom;
}

inline double silu(double z) { return z / (1.0 + std::exp(-z)); }

struct StateBase {
  or_config c;
  or_weights w;
  int batch, max_seq, kv_round;
  std::vector<int> pos;
  std::vector<double> last_q, last_k;  // [layer][batch][heads*head_dim] of the last token
  virtual ~StateBase() {}
  virtual int forward(const int32_t* tokens, int T, float* logits_f32, double* logits_f64, bool all_logits) = 0;
  virtual void set_cache(const uint16_t* kv, int length) = 0;
  virtual void get_cache(uint16_t* kv, int length) const = 0;
};

template <class A>
struct State : StateBase {
  using T = A;
  std::vector<T> cache;  // [layer][2][b][kvh][max_seq][hd]

  size_t cidx(int l, int kind, int b, int h, int p) const {
    return ((((size_t)l * 2 + kind) * batch + b) * c.n_kv_heads + h) * (size_t)max_seq * c.head_dim +
           (size_t)p * c.head_dim;
  }

  T kv_store(double v) const {
    if (!kv_round) return (T)v;
    uint16_t b = float_to_bf16_bits((float)v);
    return (T)bf16_to_double(b);
  }

  void set_cache(const uint16_t* kv, int length) override {
    for (int l = 0; l < c.n_layers; ++l)
      for (int kind = 0; kind < 2; ++kind)
        for (int b = 0; b < batch; ++b)
          for (int h = 0; h < c.n_kv_heads; ++h)
            for (int p = 0; p < length; ++p)
              for (int t = 0; t < c.head_dim; ++t) {
                size_t src = ((((((size_t)l * 2 + kind) * batch + b) * c.n_kv_heads + h) * length + p) *
                              c.head_dim) + t;
                cache[cidx(l, kind, b, h, p) + t] = (T)bf16_to_double(kv[src]);
              }
    for (int b = 0; b < batch; ++b) pos[b] = length;
  }

  void get_cache(uint16_t* kv, int length) const override {
    for (int l = 0; l < c.n_layers; ++l)
      for (int kind = 0; kind < 2; ++kind)
        for (int b = 0; b < batch; ++b)
          for (int h = 0; h < c.n_kv_heads; ++h)
            for (int p = 0; p < length; ++p)
              for (int t = 0; t < c.head_dim; ++t) {
                size_t dst = ((((((size_t)l * 2 + kind) * batch + b) * c.n_kv_heads + h) * length + p) *
                              c.head_dim) + t;
                kv[dst] = float_to_bf16_bits((float)cache[cidx(l, kind, b, h, p) + t]);
              }
  }

  // Run T tokens of every sequence through the decoder starting at pos[b]; tokens [b][T].
  // Writes logits of the last token (or of every token when all_logits) in f32 and/or f64.
  int forward(const int32_t* tokens, int ntok, float* lf32, double* lf64, bool all_logits) override {
    const int T_ = ntok;
    const int H = c.hidden, D = c.head_dim, nq = c.n_q_heads, nkv = c.n_kv_heads, F = c.ffn, V = c.vocab;
    const int N = batch * T_;  // vectors in flight, row n = b*T + t
    const bool f32_table = sizeof(T) == sizeof(float);
    for (int b = 0; b < batch; ++b) {
      if (pos[b] + T_ > max_seq) return -3;
      for (int t = 0; t < T_; ++t)
        if (tokens[b * T_ + t] < 0 || tokens[b * T_ + t] >= V) return -4;
    }
    std::vector<T> x((size_t)N * H), xn((size_t)N * H), q((size_t)N * nq * D), k((size_t)N * nkv * D),
        v((size_t)N * nkv * D), o((size_t)N * nq * D), y((size_t)N * H), g((size_t)N * F), u((size_t)N * F),
        hbuf((size_t)N * F);
    // embedding
    for (int n = 0; n < N; ++n)
      for (int i = 0; i < H; ++i) x[(size_t)n * H + i] = (T)bf16_to_double(w.embed[(size_t)tokens[n] * H + i]);
    const double scale = 1.0 / std::sqrt((double)D);
    for (int l = 0; l < c.n_layers; ++l) {
      for (int n = 0; n < N; ++n) rmsnorm(&x[(size_t)n * H], w.attn_norm[l], H, c.rms_eps, &xn[(size_t)n * H]);
      linear(w.wq[l], nq * D, H, xn.data(), N, q.data());
      linear(w.wk[l], nkv * D, H, xn.data(), N, k.data());
      linear(w.wv[l], nkv * D, H, xn.data(), N, v.data());
      if (w.q_norm_w) {
        for (int n = 0; n < N; ++n) {
          for (int h = 0; h < nq; ++h) {
            T* qh = &q[((size_t)n * nq + h) * D];
            layernorm(qh, w.q_norm_w[l] + (size_t)h * D, w.q_norm_b[l] + (size_t)h * D, D, c.rms_eps, qh);
          }
          for (int h = 0; h < nkv; ++h) {
            T* kh = &k[((size_t)n * nkv + h) * D];
            layernorm(kh, w.k_norm_w[l] + (size_t)h * D, w.k_norm_b[l] + (size_t)h * D, D, c.rms_eps, kh);
          }
        }
      }
      for (int b = 0; b < batch; ++b)
        for (int t = 0; t < T_; ++t) {
          int n = b * T_ + t, p = pos[b] + t;
          for (int h = 0; h < nq; ++h) rope_head(&q[((size_t)n * nq + h) * D], D, p, c.rope_theta, f32_table);
          for (int h = 0; h < nkv; ++h) rope_head(&k[((size_t)n * nkv + h) * D], D, p, c.rope_theta, f32_table);
          if (t == T_ - 1) {
            for (int e = 0; e < nq * D; ++e)
              last_q[((size_t)l * batch + b) * nq * D + e] = (double)q[(size_t)n * nq * D + e];
            for (int e = 0; e < nkv * D; ++e)
              last_k[((size_t)l * batch + b) * nkv * D + e] = (double)k[(size_t)n * nkv * D + e];
          }
          for (int h = 0; h < nkv; ++h) {
            for (int e = 0; e < D; ++e) {
              cache[cidx(l, 0, b, h, p) + e] = kv_store((double)k[((size_t)n * nkv + h) * D + e]);
              cache[cidx(l, 1, b, h, p) + e] = kv_store((double)v[((size_t)n * nkv + h) * D + e]);
            }
          }
        }
      // attention: token t of sequence b attends to positions 0 .. pos[b]+t (causal)
      parallel_rows(N * nq, 1LL << 16, [&](int lo, int hi) {
        for (int idx = lo; idx < hi; ++idx) {
          int n = idx / nq, h = idx % nq, b = n / T_, t = n % T_;
          int kvh = (int)((long long)h * nkv / nq);
          int L = pos[b] + t + 1;
          attend(&q[((size_t)n * nq + h) * D], &cache[cidx(l, 0, b, kvh, 0)], &cache[cidx(l, 1, b, kvh, 0)], L, D,
                 scale, &o[((size_t)n * nq + h) * D], nullptr);
        }
      });
      linear(w.wo[l], H, nq * D, o.data(), N, y.data());
      for (size_t i = 0; i < x.size(); ++i) x[i] = (T)((double)x[i] + (double)y[i]);
      for (int n = 0; n < N; ++n) rmsnorm(&x[(size_t)n * H], w.mlp_norm[l], H, c.rms_eps, &xn[(size_t)n * H]);
      linear(w.wg[l], F, H, xn.data(), N, g.data());
      linear(w.wu[l], F, H, xn.data(), N, u.data());
      for (size_t i = 0; i < hbuf.size(); ++i) hbuf[i] = (T)(silu((double)g[i]) * (double)u[i]);
      linear(w.wd[l], H, F, hbuf.data(), N, y.data());
      for (size_t i = 0; i < x.size(); ++i) x[i] = (T)((double)x[i] + (double)y[i]);
    }
    // final norm + LM head, for the last token of each sequence (or every token)
    std::vector<int> rows;
    for (int b = 0; b < batch; ++b)
      for (int t = 0; t < T_; ++t)
        if (all_logits || t == T_ - 1) rows.push_back(b * T_ + t);
    std::vector<T> xf(rows.size() * (size_t)H), lg(rows.size() * (size_t)V);
    for (size_t r = 0; r < rows.size(); ++r) rmsnorm(&x[(size_t)rows[r] * H], w.final_norm, H, c.rms_eps, &xf[r * H]);
    linear(w.lm_head, V, H, xf.data(), (int)rows.size(), lg.data());
    for (size_t i = 0; i < lg.size(); ++i) {
      if (lf32) lf32[i] = (float)lg[i];
      if (lf64) lf64[i] = (double)lg[i];
    }
    for (int b = 0; b < batch; ++b) pos[b] += T_;
    return 0;
  }
};

}  // namespace

struct or_state {
  StateBase* impl;
};

extern "C" {

void or_set_threads(int n) { g_threads = n; }

or_state* or_create(const or_config* cfg, const or_weights* w, int batch, int max_seq, int f64, int kv_round) {
  if (!cfg || !w || batch < 1 || max_seq < 1) return nullptr;
  if ((w->q_norm_w || w->q_norm_b || w->k_norm_w || w->k_norm_b) &&
      !(w->q_norm_w && w->q_norm_b && w->k_norm_w && w->k_norm_b))
    return nullptr;  // QK-norm needs all four arrays
  if (cfg->n_layers < 1 || cfg->hidden < 1 || cfg->n_q_heads < 1 || cfg->n_kv_heads < 1 || cfg->head_dim < 2 ||
      (cfg->head_dim & 1) || cfg->ffn < 1 || cfg->vocab < 1 || cfg->n_q_heads % cfg->n_kv_heads)
    return nullptr;
  StateBase* s;
  if (f64) {
    auto* t = new State<double>();
    t->cache.assign((size_t)cfg->n_layers * 2 * batch * cfg->n_kv_heads * max_seq * cfg->head_dim, 0.0);
    s = t;
  } else {
    auto* t = new State<float>();
    t->cache.assign((size_t)cfg->n_layers * 2 * batch * cfg->n_kv_heads * max_seq * cfg->head_dim, 0.0f);
    s = t;
  }
  s->c = *cfg;
  s->w = *w;
  s->batch = batch;
  s->max_seq = max_seq;
  s->kv_round = kv_round;
  s->pos.assign(batch, 0);
  s->last_q.assign((size_t)cfg->n_layers * batch * cfg->n_q_heads * cfg->head_dim, 0.0);
  s->last_k.assign((size_t)cfg->n_layers * batch * cfg->n_kv_heads * cfg->head_dim, 0.0);
  return new or_state{s};
}

void or_destroy(or_state* s) {
  if (!s) return;
  delete s->impl;
  delete s;
}

int or_prefill(or_state* s, const int32_t* tokens, int T, float* last_logits) {
  if (!s || !tokens || T < 1) return -1;
  return s->impl->forward(tokens, T, last_logits, nullptr, false);
}

int or_decode(or_state* s, const int32_t* tokens, float* logits) {
  if (!s || !tokens || !logits) return -1;
  return s->impl->forward(tokens, 1, logits, nullptr, false);
}

int or_decode_f64(or_state* s, const int32_t* tokens, double* logits) {
  if (!s || !tokens || !logits) return -1;
  return s->impl->forward(tokens, 1, nullptr, logits, false);
}

int or_set_cache(or_state* s, const uint16_t* kv, int length) {
  if (!s || !kv || length < 0 || length > s->impl->max_seq) return -1;
  s->impl->set_cache(kv, length);
  return 0;
}

int or_get_cache(const or_state* s, uint16_t* kv, int length) {
  if (!s || !kv || length < 0 || length > s->impl->max_seq) return -1;
  s->impl->get_cache(kv, length);
  return 0;
}

int or_set_positions(or_state* s, const int32_t* pos) {
  if (!s || !pos) return -1;
  for (int b = 0; b < s->impl->batch; ++b)
    if (pos[b] < 0 || pos[b] > s->impl->max_seq) return -1;
  for (int b = 0; b < s->impl->batch; ++b) s->impl->pos[b] = pos[b];
  return 0;
}

int or_position(const or_state* s, int b) {
  if (!s || b < 0 || b >= s->impl->batch) return -1;
  return s->impl->pos[b];
}

int or_get_qk(const or_state* s, int layer, double* q, double* k) {
  if (!s || !q || !k || layer < 0 || layer >= s->impl->c.n_layers) return -1;
  const StateBase* b = s->impl;
  const size_t nq = (size_t)b->batch * b->c.n_q_heads * b->c.head_dim;
  const size_t nk = (size_t)b->batch * b->c.n_kv_heads * b->c.head_dim;
  std::memcpy(q, b->last_q.data() + (size_t)layer * nq, nq * sizeof(double));
  std::memcpy(k, b->last_k.data() + (size_t)layer * nk, nk * sizeof(double));
  return 0;
}

int or_argmax(const float* logits, int n) {
  int best = 0;
  for (int i = 1; i < n; ++i)
    if (logits[i] > logits[best]) best = i;
  return best;
}

void or_rmsnorm(const double* x, const double* g, int n, double eps, double* y) {
  double ss = 0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double r = 1.0 / std::sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) y[i] = x[i] * r * g[i];
}

void or_layernorm(const double* x, const double* g, const double* b, int n, double eps, double* y) {
  double sum = 0;
  for (int i = 0; i < n; ++i) sum += x[i];
  const double mean = sum / n;
  double sq = 0;
  for (int i = 0; i < n; ++i) sq += (x[i] - mean) * (x[i] - mean);
  const double r = 1.0 / std::sqrt(sq / n + eps);
  for (int i = 0; i < n; ++i) y[i] = (x[i] - mean) * r * g[i] + b[i];
}

void or_matvec_bf16(const uint16_t* W, const double* x, int rows, int cols, double* y) {
  linear<double>(W, rows, cols, x, 1, y);
}

void or_rope(double* v, int head_dim, int pos, double theta) { rope_head<double>(v, head_dim, pos, theta, false); }

void or_rope_cos_sin(int head_dim, int pos, double theta, float* cos_out, float* sin_out) {
  for (int i = 0; i < head_dim / 2; ++i) {
    double c, s;
    rope_angle(head_dim, pos, theta, i, &c, &s);
    cos_out[i] = (float)c;
    sin_out[i] = (float)s;
  }
}

void or_attention_head(const double* q, const double* k, const double* v, int L, int d, double scale, double* o,
                       double* probs) {
  attend<double, double>(q, k, v, L, d, scale, o, probs);
}

double or_silu(double z) { return silu(z); }

int or_attention_decode_f16(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, int BH, int d, int L,
                            double scale, double* o) {
  if (!q || !k_t || !v || !o || BH < 1 || d < 1 || L < 1) return -1;
  parallel_rows(BH, (long long)L * d * 2, [&](int lo, int hi) {
    std::vector<double> qq(d), kk((size_t)L * d), vv((size_t)L * d);
    for (int bh = lo; bh < hi; ++bh) {
      for (int t = 0; t < d; ++t) qq[t] = f16_to_double(q[(size_t)bh * d + t]);
      // K arrives transposed ([d][L], key index fastest): gather key rows
      for (int t = 0; t < d; ++t)
        for (int j = 0; j < L; ++j) kk[(size_t)j * d + t] = f16_to_double(k_t[((size_t)bh * d + t) * L + j]);
      for (size_t i = 0; i < (size_t)L * d; ++i) vv[i] = f16_to_double(v[(size_t)bh * L * d + i]);
      attend<double, double>(qq.data(), kk.data(), vv.data(), L, d, scale, o + (size_t)bh * d, nullptr);
    }
  });
  return 0;
}

}  // extern "C"
