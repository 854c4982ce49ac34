// CPU oracle for the DeepSeek Sparse Attention (DSA) hot path, in plain C++.
//
// TEST INFRASTRUCTURE ONLY. It is called by the tests, by the smoke check and
// by the benchmark's CPU legs (through oracle/dsa_oracle.py); the product path
// never calls it. It shares no code, header, table or constant with the CUDA
// library under sparse_long_context_04_b200/ and includes nothing from it.
//
// Every value is computed in double precision by the plain definition, one
// query row at a time: loops in the order the definition sums, no blocking, no
// library kernels. Independent query rows run on separate std::threads; nothing
// else is parallel, so each row's arithmetic is the same whatever the thread
// count.
//
// Sources (the DeepSeek-V3.2-Exp pages; none prints an equation, so each stage
// is written from the words):
//   [jdon-indexer]   jdon.com "DeepSeek-V3.2-Exp", paragraph introducing the
//                    lightning indexer: light enough for FP8, very few heads,
//                    each query token scored against each earlier token by a
//                    weighted sum of ReLU-activated dot products.
//   [jdon-matchmake] same page, the "matchmaking" analogy paragraph: ReLU on the
//                    q_I / k_I meeting score, w_I as the weight, the highest
//                    scores form the top-k set.
//   [jdon-sparse]    same page, sparse-training paragraph: each query keeps the
//                    2048 (K = 2048) highest-scoring earlier tokens; the main model
//                    trains on the selected entries only.
//   [jdon-select]    same page, fine-grained selection paragraph: only the chosen
//                    key/value entries take part; the output hidden state u_t.
//   [jdon-warmup]    same page, warm-up paragraph: the indexer copies the main
//                    attention's distribution through a KL-divergence loss.
//   [openi-mla]      openi.cn "DeepSeek-V3.2", technical section: indexer scores
//                    against earlier tokens, top-k value entries, MLA in MQA mode
//                    (one latent entry shared by every query head).
//   [mundobytes-run] mundobytes.com "Deepseek-v3-2-exp", run guide: the serving
//                    command uses 64-token KV pages; open-kernels paragraph: the
//                    indexer kernels come in a paged version.
//
// Readings where the pages are silent (each function repeats the one it uses):
//   * I[t,s] = sum_j w[t,j] * max(0, q_I[t,j] . k_I[s]): ReLU per head on the dot
//     product, then the weighted sum over heads. FP8 inputs are e4m3 bytes with
//     one positive fp32 scale per token, multiplying the decoded vector.
//   * causal set s <= pos_t, the query's own position included.
//   * selection order: score descending, then position ascending; -0 == +0; NaN
//     below every number; emitted in ascending position, -1 padded to k.
//   * attention: key = the whole latent row (Dk values), value = its first Dv
//     values, one row shared by all heads; plain softmax with the caller's scale.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ------------------------------------------------------------------ number formats

// OCP FP8 E4M3 ("e4m3fn") from its bit fields: sign, 4 exponent bits with bias 7,
// 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no
// infinities.
double e4m3_value(unsigned byte) {
  const unsigned s = (byte >> 7) & 1u, e = (byte >> 3) & 0xFu, m = byte & 7u;
  if (e == 0xFu && m == 7u) return std::numeric_limits<double>::quiet_NaN();
  double mag;
  if (e == 0)
    mag = (m / 8.0) * std::ldexp(1.0, -6);
  else
    mag = (1.0 + m / 8.0) * std::ldexp(1.0, (int)e - 7);
  return s ? -mag : mag;
}

// The 256 values of e4m3_value, listed once (decoding is then a lookup).
const double *e4m3_table() {
  static const std::vector<double> table = [] {
    std::vector<double> v(256);
    for (unsigned b = 0; b < 256; ++b) v[b] = e4m3_value(b);
    return v;
  }();
  return table.data();
}

// bfloat16 is the upper half of an IEEE binary32.
double bf16_value(uint16_t bits) {
  const uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

float f32_at(const uint8_t *p) {  // little-endian binary32 stored in a byte array
  float f;
  std::memcpy(&f, p, 4);
  return f;
}

// Byte of the e4m3 value nearest to y, ties to the even code, saturating at
// +-448, NaN -> 0x7F. The codes 0x00..0x7E are the finite magnitudes in
// increasing order, so rounding is a search among them.
uint8_t encode_e4m3(double y) {
  if (std::isnan(y)) return 0x7F;
  const double a = std::min(std::fabs(y), 448.0);
  unsigned hi = 0;  // first code whose magnitude is >= a
  while (hi < 126 && e4m3_value(hi) < a) ++hi;
  const unsigned lo = hi > 0 ? hi - 1 : 0;
  const double d_lo = a - e4m3_value(lo), d_hi = e4m3_value(hi) - a;
  const bool take_hi = d_hi < d_lo || (d_hi == d_lo && hi != lo && (hi % 2) == 0);
  unsigned code = take_hi ? hi : lo;
  if (std::signbit(y)) code |= 0x80u;
  return (uint8_t)code;
}

// ------------------------------------------------------------------ a workload
struct Case {
  int fp8;                 // 1: e4m3 indexer + bf16 attention; 0: all float32
  int B, T;
  int H_I, d_I, H, Dk, Dv, k;
  double softmax_scale;
  const int32_t *seq_lens;  // [B]
  const int32_t *pos;       // [T]  position of each query row
  const int32_t *row_seq;   // [T]  sequence of each query row
  const void *q_idx;        // fp8: uint8 [T][H_I][d_I]; else float [T][H_I][d_I]
  const float *q_scale;     // fp8: [T]
  const float *w;           // [T][H_I]
  const void *q;            // fp8: bf16 bits [T][H][Dk]; else float
  int page_size;            // 0: contiguous caches; else paged with this page size
  int n_max;                // contiguous row stride of the caches
  const void *k_idx;        // contiguous: [B][n_max][d_I] (uint8 or float)
  const float *k_scale;     // contiguous fp8: [B][n_max]
  const uint8_t *k_pages;   // paged: [pages][page_size*d_I + 4*page_size]
  const int32_t *page_table;
  int max_pages;
  const void *kv;           // contiguous [B][n_max][Dk]; paged [pages*page_size][Dk]
};

// Dequantised indexer key of position s of sequence b (paged: page from the page
// table, slot s % page_size; an indexer page is page_size key rows of d_I bytes
// followed by page_size little-endian fp32 scales) [mundobytes-run].
void indexer_key(const Case &c, int b, int s, double *out) {
  if (!c.fp8) {
    const float *k = (const float *)c.k_idx + ((size_t)b * c.n_max + s) * c.d_I;
    for (int d = 0; d < c.d_I; ++d) out[d] = k[d];
    return;
  }
  const uint8_t *codes;
  double scale;
  if (c.page_size == 0) {
    codes = (const uint8_t *)c.k_idx + ((size_t)b * c.n_max + s) * c.d_I;
    scale = c.k_scale[(size_t)b * c.n_max + s];
  } else {
    const int P = c.page_size;
    const int page = c.page_table[(size_t)b * c.max_pages + s / P];
    const uint8_t *pg = c.k_pages + (size_t)page * ((size_t)P * c.d_I + 4 * (size_t)P);
    codes = pg + (size_t)(s % P) * c.d_I;
    scale = f32_at(pg + (size_t)P * c.d_I + 4 * (size_t)(s % P));
  }
  const double *dec = e4m3_table();
  for (int d = 0; d < c.d_I; ++d) out[d] = scale * dec[codes[d]];
}

// Latent row of position s of sequence b, Dk values [openi-mla].
void latent_row(const Case &c, int b, int s, double *out) {
  size_t r;
  if (c.page_size == 0) {
    r = (size_t)b * c.n_max + s;
  } else {
    const int P = c.page_size;
    r = (size_t)c.page_table[(size_t)b * c.max_pages + s / P] * P + s % P;
  }
  if (c.fp8) {
    const uint16_t *v = (const uint16_t *)c.kv + r * c.Dk;
    for (int d = 0; d < c.Dk; ++d) out[d] = bf16_value(v[d]);
  } else {
    const float *v = (const float *)c.kv + r * c.Dk;
    for (int d = 0; d < c.Dk; ++d) out[d] = v[d];
  }
}

// Indexer query heads [H_I][d_I] (dequantised) of row t.
void indexer_query(const Case &c, int t, double *out) {
  const size_t n = (size_t)c.H_I * c.d_I;
  if (c.fp8) {
    const uint8_t *q = (const uint8_t *)c.q_idx + (size_t)t * n;
    const double s = c.q_scale[t];
    const double *dec = e4m3_table();
    for (size_t i = 0; i < n; ++i) out[i] = s * dec[q[i]];
  } else {
    const float *q = (const float *)c.q_idx + (size_t)t * n;
    for (size_t i = 0; i < n; ++i) out[i] = q[i];
  }
}

// Query heads [H][Dk] of row t.
void attn_query(const Case &c, int t, double *out) {
  const size_t n = (size_t)c.H * c.Dk;
  if (c.fp8) {
    const uint16_t *q = (const uint16_t *)c.q + (size_t)t * n;
    for (size_t i = 0; i < n; ++i) out[i] = bf16_value(q[i]);
  } else {
    const float *q = (const float *)c.q + (size_t)t * n;
    for (size_t i = 0; i < n; ++i) out[i] = q[i];
  }
}

// ------------------------------------------------------------------ the three stages

// Stage 1 [jdon-indexer], [jdon-matchmake]: score of one key against one query
// token: sum over heads j of w[j] * max(0, q[j] . key).
double indexer_score(const double *q, const double *w, const double *key, int H_I, int d_I) {
  double acc = 0.0;
  for (int j = 0; j < H_I; ++j) {
    double dot = 0.0;
    for (int d = 0; d < d_I; ++d) dot += q[(size_t)j * d_I + d] * key[d];
    acc += w[j] * (dot > 0.0 ? dot : 0.0);
  }
  return acc;
}

// Stage 2 [jdon-sparse], [jdon-select]: the min(k, n) positions that come first
// under (score descending, position ascending) with -0 == +0 and NaN lowest,
// listed in ascending position, then -1 up to k.
bool ranks_before(float va, int sa, float vb, int sb) {
  const bool na = std::isnan(va), nb = std::isnan(vb);
  if (na != nb) return nb;            // a number before NaN
  if (!na && va != vb) return va > vb;  // -0.0 == +0.0 here
  return sa < sb;
}

void topk_row(const float *scores, int n, int k, int32_t *out) {
  std::vector<int> order(n);
  for (int s = 0; s < n; ++s) order[s] = s;
  const int m = std::min(k, n);
  auto cmp = [&](int a, int b) { return ranks_before(scores[a], a, scores[b], b); };
  if (m < n) std::nth_element(order.begin(), order.begin() + m, order.end(), cmp);
  std::sort(order.begin(), order.begin() + m);
  for (int i = 0; i < m; ++i) out[i] = order[i];
  for (int i = m; i < k; ++i) out[i] = -1;
}

// Stage 3 [jdon-select], [openi-mla]: for each head h, z_s = scale * q[h] . row_s
// over the m selected rows; o[h] = sum_s softmax(z)_s row_s[0:Dv];
// lse[h] = log sum_s exp z_s. Two passes: the maximum, then the exponentials.
// No selected row: o = 0, lse = -inf.
void sparse_attn(const double *q, const double *rows, int m, int H, int Dk, int Dv, double scale, double *o,
                 double *lse) {
  std::vector<double> z(m > 0 ? m : 1);
  for (int h = 0; h < H; ++h) {
    double *oh = o + (size_t)h * Dv;
    for (int d = 0; d < Dv; ++d) oh[d] = 0.0;
    if (m == 0) {
      lse[h] = -std::numeric_limits<double>::infinity();
      continue;
    }
    double zmax = -std::numeric_limits<double>::infinity();
    for (int s = 0; s < m; ++s) {
      double dot = 0.0;
      for (int d = 0; d < Dk; ++d) dot += q[(size_t)h * Dk + d] * rows[(size_t)s * Dk + d];
      z[s] = scale * dot;
      zmax = std::max(zmax, z[s]);
    }
    double Z = 0.0;
    for (int s = 0; s < m; ++s) {
      const double p = std::exp(z[s] - zmax);
      Z += p;
      for (int d = 0; d < Dv; ++d) oh[d] += p * rows[(size_t)s * Dk + d];
    }
    for (int d = 0; d < Dv; ++d) oh[d] /= Z;
    lse[h] = zmax + std::log(Z);
  }
}

// ------------------------------------------------------------------ threads over rows
template <typename F>
void for_rows(int nrows, int threads, F f) {
  if (threads <= 0) threads = (int)std::max(1u, std::thread::hardware_concurrency());
  threads = std::max(1, std::min(threads, nrows));
  if (threads == 1) {
    for (int r = 0; r < nrows; ++r) f(r);
    return;
  }
  std::atomic<int> next(0);
  std::vector<std::thread> pool;
  for (int i = 0; i < threads; ++i)
    pool.emplace_back([&] {
      for (int r = next++; r < nrows; r = next++) f(r);
    });
  for (auto &th : pool) th.join();
}

// Scores of row t over s = 0..pos_t into out[0..pos_t].
void row_scores(const Case &c, int t, double *out) {
  const int b = c.row_seq[t], pos = c.pos[t];
  std::vector<double> q((size_t)c.H_I * c.d_I), key(c.d_I);
  indexer_query(c, t, q.data());
  const double *w = nullptr;
  std::vector<double> wd(c.H_I);
  for (int j = 0; j < c.H_I; ++j) wd[j] = c.w[(size_t)t * c.H_I + j];
  w = wd.data();
  for (int s = 0; s <= pos; ++s) {
    indexer_key(c, b, s, key.data());
    out[s] = indexer_score(q.data(), w, key.data(), c.H_I, c.d_I);
  }
}

// Attention of row t over the selected positions idx[0..k) (-1 = padding).
void row_attention(const Case &c, int t, const int32_t *idx, double *o, double *lse) {
  const int b = c.row_seq[t];
  std::vector<int> sel;
  for (int i = 0; i < c.k; ++i)
    if (idx[i] >= 0) sel.push_back(idx[i]);
  std::vector<double> q((size_t)c.H * c.Dk), rows((size_t)(sel.empty() ? 1 : sel.size()) * c.Dk);
  attn_query(c, t, q.data());
  for (size_t i = 0; i < sel.size(); ++i) latent_row(c, b, sel[i], rows.data() + i * c.Dk);
  sparse_attn(q.data(), rows.data(), (int)sel.size(), c.H, c.Dk, c.Dv, c.softmax_scale, o, lse);
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

typedef Case oracle_case;

int oracle_hardware_threads(void) { return (int)std::max(1u, std::thread::hardware_concurrency()); }

double oracle_e4m3_value(unsigned byte) { return e4m3_value(byte & 0xFFu); }
double oracle_bf16_value(unsigned bits) { return bf16_value((uint16_t)bits); }

void oracle_decode_e4m3(const uint8_t *b, long long n, double *out) {
  for (long long i = 0; i < n; ++i) out[i] = e4m3_value(b[i]);
}

void oracle_decode_bf16(const uint16_t *b, long long n, double *out) {
  for (long long i = 0; i < n; ++i) out[i] = bf16_value(b[i]);
}

// x~ = s * dec(b) for rows of `cols` e4m3 bytes with one scale per row.
void oracle_dequant(const uint8_t *b, long long rows, long long cols, const float *scale, double *out) {
  for (long long r = 0; r < rows; ++r)
    for (long long i = 0; i < cols; ++i) out[r * cols + i] = (double)scale[r] * e4m3_value(b[r * cols + i]);
}

void oracle_encode_e4m3(const double *y, long long n, uint8_t *out) {
  for (long long i = 0; i < n; ++i) out[i] = encode_e4m3(y[i]);
}

// Per-token quantisation of one indexer key row, in fp32 as a kernel computes it
// (the integer code is decided by float arithmetic, so both sides take it in
// fp32): scale = float(max|x|) / 448 (1 for an all-zero row), y = float(x) / scale,
// code = nearest e4m3 to y, ties to even [jdon-indexer], [mundobytes-run].
void oracle_quantize_key_row(const float *x, int d, uint8_t *codes, float *scale) {
  float amax = 0.0f;
  for (int i = 0; i < d; ++i) amax = std::max(amax, std::fabs(x[i]));
  const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
  for (int i = 0; i < d; ++i) {
    const float y = x[i] / sc;
    codes[i] = encode_e4m3((double)y);
  }
  *scale = sc;
}

// Stage 1 on raw float64 arrays: q [H_I][d_I], w [H_I], keys [n][d_I] -> out [n].
void oracle_indexer_row(const double *q, const double *w, const double *keys, long long n, int H_I, int d_I,
                        double *out) {
  for (long long s = 0; s < n; ++s) out[s] = indexer_score(q, w, keys + s * d_I, H_I, d_I);
}

void oracle_topk_row(const float *scores, int n, int k, int32_t *out) { topk_row(scores, n, k, out); }

// Stage 2 over many rows: row r has n[r] scores at scores + r*ld.
void oracle_topk_rows(const float *scores, long long ld, const int32_t *n, int nrows, int k, int32_t *out,
                      int threads) {
  for_rows(nrows, threads, [&](int r) { topk_row(scores + (size_t)r * ld, n[r], k, out + (size_t)r * k); });
}

// Stage 3 on raw float64 arrays: q [H][Dk], rows [m][Dk] -> o [H][Dv], lse [H].
void oracle_sparse_attn_row(const double *q, const double *rows, int m, int H, int Dk, int Dv, double scale,
                            double *o, double *lse) {
  sparse_attn(q, rows, m, H, Dk, Dv, scale, o, lse);
}

// Logical views of a sequence's caches: indexer keys [len][d_I], latent rows [len][Dk].
void oracle_seq_keys(const oracle_case *c, int b, double *k_out, double *kv_out) {
  const int L = c->seq_lens[b];
  for (int s = 0; s < L; ++s) {
    if (k_out) indexer_key(*c, b, s, k_out + (size_t)s * c->d_I);
    if (kv_out) latent_row(*c, b, s, kv_out + (size_t)s * c->Dk);
  }
}

// Row t's indexer query heads [H_I][d_I], weights [H_I] and query heads [H][Dk].
void oracle_query_row(const oracle_case *c, int t, double *qI, double *w, double *q) {
  if (qI) indexer_query(*c, t, qI);
  if (w)
    for (int j = 0; j < c->H_I; ++j) w[j] = c->w[(size_t)t * c->H_I + j];
  if (q) attn_query(*c, t, q);
}

// Stage 1 for query rows rows[0..nrows): out[r*ld + s], s = 0..pos.
void oracle_indexer_rows(const oracle_case *c, const int32_t *rows, int nrows, double *out, long long ld,
                         int threads) {
  for_rows(nrows, threads, [&](int r) { row_scores(*c, rows[r], out + (size_t)r * ld); });
}

// Stage 3 for query rows on given selections idx [nrows][k]: o [nrows][H][Dv], lse [nrows][H].
void oracle_attn_rows(const oracle_case *c, const int32_t *rows, int nrows, const int32_t *idx, double *o,
                      double *lse, int threads) {
  for_rows(nrows, threads, [&](int r) {
    row_attention(*c, rows[r], idx + (size_t)r * c->k, o + (size_t)r * c->H * c->Dv, lse + (size_t)r * c->H);
  });
}

// The whole path for query rows: scores (optional, double, out[r*ld + s]), the
// selection on the scores rounded to float32, and the attention on it.
void oracle_forward_rows(const oracle_case *c, const int32_t *rows, int nrows, double *scores, long long ld,
                         int32_t *idx, double *o, double *lse, int threads) {
  for_rows(nrows, threads, [&](int r) {
    const int t = rows[r], n = c->pos[t] + 1;
    std::vector<double> sc(n);
    row_scores(*c, t, sc.data());
    std::vector<float> s32(n);
    for (int s = 0; s < n; ++s) s32[s] = (float)sc[s];
    int32_t *ix = idx + (size_t)r * c->k;
    topk_row(s32.data(), n, c->k, ix);
    row_attention(*c, t, ix, o + (size_t)r * c->H * c->Dv, lse + (size_t)r * c->H);
    if (scores)
      for (int s = 0; s < n; ++s) scores[(size_t)r * ld + s] = sc[s];
  });
}

// Cache write [mundobytes-run], [jdon-indexer]: row t's new indexer key, quantised
// per token, and its latent row (bf16 bits, copied) go to the row's own position
// pos_t of its sequence. Paged: k_cache [pages][P*d_I + 4P] (codes, then scales),
// kv_cache [pages*P][Dk]; contiguous: k_cache [B][n_max][d_I] with k_scale
// [B][n_max], kv_cache [B][n_max][Dk]. Updated in place.
void oracle_cache_append(const oracle_case *c, const float *k_new, const uint16_t *kv_new, uint8_t *k_cache,
                         float *k_scale, uint16_t *kv_cache) {
  const int P = c->page_size, d_I = c->d_I;
  std::vector<uint8_t> codes(d_I);
  for (int t = 0; t < c->T; ++t) {
    const int b = c->row_seq[t], pos = c->pos[t];
    float sc;
    oracle_quantize_key_row(k_new + (size_t)t * d_I, d_I, codes.data(), &sc);
    size_t kv_row;
    if (P) {
      const size_t page = (size_t)c->page_table[(size_t)b * c->max_pages + pos / P];
      uint8_t *pg = k_cache + page * ((size_t)P * d_I + 4 * (size_t)P);
      std::memcpy(pg + (size_t)(pos % P) * d_I, codes.data(), d_I);
      std::memcpy(pg + (size_t)P * d_I + 4 * (size_t)(pos % P), &sc, 4);
      kv_row = page * P + pos % P;
    } else {
      const size_t r = (size_t)b * c->n_max + pos;
      std::memcpy(k_cache + r * d_I, codes.data(), d_I);
      k_scale[r] = sc;
      kv_row = r;
    }
    if (kv_new) std::memcpy(kv_cache + kv_row * c->Dk, kv_new + (size_t)t * c->Dk, 2 * (size_t)c->Dk);
  }
}

// Indexer loss on the selected set [jdon-warmup], [jdon-sparse]: for one query
// row over its m selected rows, the target p = the heads' attention over the set
// averaged over the H heads (each head's softmax sums to 1), the indexer's
// distribution r = softmax of the m scores, loss = sum p (log p - log r) over
// p > 0, grad = r - p (d loss / d scores). Returns the loss.
double oracle_indexer_kl_row(const double *q, const double *rows, int m, int H, int Dk, double scale,
                             const double *scores, double *p_out, double *grad) {
  std::vector<double> p(m, 0.0), z(m);
  for (int h = 0; h < H; ++h) {
    double zmax = -std::numeric_limits<double>::infinity();
    for (int s = 0; s < m; ++s) {
      double dot = 0.0;
      for (int d = 0; d < Dk; ++d) dot += q[(size_t)h * Dk + d] * rows[(size_t)s * Dk + d];
      z[s] = scale * dot;
      zmax = std::max(zmax, z[s]);
    }
    double Z = 0.0;
    for (int s = 0; s < m; ++s) Z += std::exp(z[s] - zmax);
    for (int s = 0; s < m; ++s) p[s] += std::exp(z[s] - zmax) / Z;
  }
  for (int s = 0; s < m; ++s) p[s] /= H;
  double smax = -std::numeric_limits<double>::infinity();
  for (int s = 0; s < m; ++s) smax = std::max(smax, scores[s]);
  double R = 0.0;
  for (int s = 0; s < m; ++s) R += std::exp(scores[s] - smax);
  double loss = 0.0;
  for (int s = 0; s < m; ++s) {
    const double r = std::exp(scores[s] - smax) / R;
    if (p[s] > 0.0) loss += p[s] * (std::log(p[s]) - std::log(r));
    if (grad) grad[s] = r - p[s];
    if (p_out) p_out[s] = p[s];
  }
  return loss;
}

// Backward of stage 3 for one query row [jdon-sparse]: gradients of sum(dO * o)
// with respect to q [H][Dk] and the m selected rows [m][Dk]. With P the per-head
// softmax, dP = dO . v, D_h = sum_s P dP: dz = P (dP - D); dq = scale dz . rows;
// drow = scale dz^T . q over all Dk, plus P^T . dO on the first Dv values.
void oracle_attn_backward_row(const double *q, const double *rows, int m, int H, int Dk, int Dv, double scale,
                              const double *dO, double *dq, double *drows) {
  for (size_t i = 0; i < (size_t)H * Dk; ++i) dq[i] = 0.0;
  for (size_t i = 0; i < (size_t)m * Dk; ++i) drows[i] = 0.0;
  if (m == 0) return;
  std::vector<double> P(m), dP(m);
  for (int h = 0; h < H; ++h) {
    const double *qh = q + (size_t)h * Dk;
    const double *g = dO + (size_t)h * Dv;
    double zmax = -std::numeric_limits<double>::infinity();
    for (int s = 0; s < m; ++s) {
      double dot = 0.0;
      for (int d = 0; d < Dk; ++d) dot += qh[d] * rows[(size_t)s * Dk + d];
      P[s] = scale * dot;
      zmax = std::max(zmax, P[s]);
    }
    double Z = 0.0;
    for (int s = 0; s < m; ++s) {
      P[s] = std::exp(P[s] - zmax);
      Z += P[s];
    }
    double D = 0.0;
    for (int s = 0; s < m; ++s) {
      P[s] /= Z;
      double dot = 0.0;
      for (int d = 0; d < Dv; ++d) dot += g[d] * rows[(size_t)s * Dk + d];
      dP[s] = dot;
      D += P[s] * dP[s];
    }
    for (int s = 0; s < m; ++s) {
      const double dz = P[s] * (dP[s] - D);
      double *dr = drows + (size_t)s * Dk;
      for (int d = 0; d < Dk; ++d) {
        dq[(size_t)h * Dk + d] += scale * dz * rows[(size_t)s * Dk + d];
        dr[d] += scale * dz * qh[d];
      }
      for (int d = 0; d < Dv; ++d) dr[d] += P[s] * g[d];
    }
  }
}

// Backward over the query rows of one sequence: q_rows [R][H][Dk], the
// sequence's latent rows by position kv [L][Dk], selections idx [R][k] (-1 =
// padding), dO [R][H][Dv]. dq [R][H][Dk]; dkv [L][Dk] sums the gradients of every
// slot that selected each position (a position selected twice counts twice).
void oracle_attn_backward_seq(const double *q_rows, const double *kv, long long L, const int32_t *idx, int R, int k,
                              int H, int Dk, int Dv, double scale, const double *dO, double *dq, double *dkv) {
  for (size_t i = 0; i < (size_t)L * Dk; ++i) dkv[i] = 0.0;
  for (int r = 0; r < R; ++r) {
    std::vector<int> sel;
    for (int i = 0; i < k; ++i)
      if (idx[(size_t)r * k + i] >= 0) sel.push_back(idx[(size_t)r * k + i]);
    double *dq_r = dq + (size_t)r * H * Dk;
    if (sel.empty()) {
      for (size_t i = 0; i < (size_t)H * Dk; ++i) dq_r[i] = 0.0;
      continue;
    }
    std::vector<double> rows(sel.size() * Dk), drows(sel.size() * Dk);
    for (size_t i = 0; i < sel.size(); ++i)
      std::memcpy(rows.data() + i * Dk, kv + (size_t)sel[i] * Dk, sizeof(double) * Dk);
    oracle_attn_backward_row(q_rows + (size_t)r * H * Dk, rows.data(), (int)sel.size(), H, Dk, Dv, scale,
                             dO + (size_t)r * H * Dv, dq_r, drows.data());
    for (size_t i = 0; i < sel.size(); ++i)
      for (int d = 0; d < Dk; ++d) dkv[(size_t)sel[i] * Dk + d] += drows[i * Dk + d];
  }
}

}  // extern "C"
