// fp64 CPU oracle of the sparse-attention layer: IndexPool -> lightning
// indexer -> top-k blocks -> softmax attention over the selected MLA latent
// rows.
//
// TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
// definition that the CUDA path is checked against.  Only the test suite,
// the smoke check and the benchmark's CPU-baseline leg may load it; the
// product path never does.  It shares no code, header, table or helper with
// the CUDA library.
//
// Sources (web pages, cited by title and section):
//  [W1] "GLM-5.3-Flash: 하이브리드 희소·선형 어텐션과 IndexPool·EPD로 1M 컨텍스트를
//       오픈 소스로 서빙하는 방법" -- sections "희소 어텐션: 인덱서로 필요한
//       토큰만" and "IndexPool: 인덱서 KV 캐시를 4배 압축" (the pooling formula).
//  [W3] "GLM-5.3 Sparse Attention은 연산량을 줄이지만 HBM 수요는 지속된다" --
//       section "GLM-5.3 Sparse Attention이 실제로 바꾸는 것" (indexer -> top-k ->
//       MLA on the selected positions; dense below the 2048-position budget).
//  [W4] "GLM-5.3-Flash vs Qwen3.8-Flash-Next: 두 중국 AI 연구소가 독립적으로 같은
//       모델 설계로 수렴한 이유" -- section "수렴점 2 — 4배 압축 후 2,048 토큰만
//       유지" (32-head indexer, top-2048, 4-token blocks x 512) and section
//       "의견이 갈리는 지점 — 위치 인코딩" (NoPE: no rotary term).
//  The indexer formula I(t,b) = sum_h w_{t,h} ReLU(q_{t,h} . k_b) is not on
//  the pages; it is the DeepSeek sparse-attention indexer form that [W3]
//  names, fixed by the workload specification.
//
// Every floating-point step is done in fp64.  The only roundings are the
// ones the method's storage formats impose: the pooled key is stored as
// bf16 (one round-to-nearest-even of the exact fp64 sum) or, in the INT8
// cache, as int8 codes of that sum (one round-half-even after an exact
// power-of-two scaling; the query heads likewise), a latent row of the
// FP8 cache is stored as E4M3 codes of the row over a power-of-two scale
// (one nearest-even rounding), and the top-k
// decision is taken on the score rounded to fp32, the precision in which
// scores are stored and ranked on the device.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

double bf16_to_f64(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// Round a finite double to the nearest bf16 (8 significant bits), ties to
// even, by scaling to an integer significand and rounding once.
uint16_t f64_to_bf16_rne(double v) {
  if (v == 0.0) return std::signbit(v) ? 0x8000 : 0x0000;
  int e = 0;
  std::frexp(std::fabs(v), &e);         // |v| = m * 2^e, m in [0.5, 1)
  int qe = e - 8;                       // weight of the last kept bit
  if (qe < -133) qe = -133;             // bf16 subnormal spacing
  double r = std::nearbyint(std::ldexp(std::fabs(v), -qe));  // exact scale
  double a = std::ldexp(r, qe);
  float f = static_cast<float>(a);      // exact: a has <= 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, 4);
  uint16_t h = static_cast<uint16_t>(u >> 16);
  if (std::signbit(v)) h |= 0x8000;
  return h;
}

int pick_threads(int nthreads) {
  if (nthreads > 0) return nthreads;
  unsigned hc = std::thread::hardware_concurrency();
  return hc ? static_cast<int>(hc) : 1;
}

}  // namespace

extern "C" {

int orc_threads(int requested) { return pick_threads(requested); }

uint16_t orc_bf16_rne(double v) { return f64_to_bf16_rne(v); }

// IndexPool cache write [W1 "IndexPool"]: block b holds tokens 4b..4b+3 in
// time order and k_pool[b] = sum_{i=0..3} w_i k[4b+i], with sum_i w_i = 1.
// Only complete blocks are pooled: n_tok / pool of them.
void orc_pool(const uint16_t* raw, int64_t n_tok, int dim, int pool,
              const double* w, uint16_t* pooled) {
  const int64_t nblk = n_tok / pool;
  for (int64_t b = 0; b < nblk; ++b) {
    for (int d = 0; d < dim; ++d) {
      double acc = 0.0;
      for (int i = 0; i < pool; ++i)
        acc += w[i] * bf16_to_f64(raw[(b * pool + i) * dim + d]);
      pooled[b * dim + d] = f64_to_bf16_rne(acc);
    }
  }
}

// IndexPool with data-dependent weights (the per-token reading of [W1
// "IndexPool"]: the learned weights come with the tokens): token p carries
// its own pooling weight wt[p], the four weights of a block sum to 1, and
// k_pool[b] = sum_{i=0..3} wt[4b+i] k[4b+i].  One fp64 sum in time order,
// one rounding to bf16, as orc_pool.
void orc_pool_tok(const uint16_t* raw, int64_t n_tok, int dim, int pool,
                  const double* wt, uint16_t* pooled) {
  const int64_t nblk = n_tok / pool;
  for (int64_t b = 0; b < nblk; ++b) {
    for (int d = 0; d < dim; ++d) {
      double acc = 0.0;
      for (int i = 0; i < pool; ++i)
        acc += wt[b * pool + i] * bf16_to_f64(raw[(b * pool + i) * dim + d]);
      pooled[b * dim + d] = f64_to_bf16_rne(acc);
    }
  }
}

// Lightning-indexer score of every pooled block against one query
// [W3 "실제로 바꾸는 것"; formula as fixed by the workload specification]:
//   s[b] = sum_h w_h * max(0, sum_d q[h][d] * k_pool[b][d]).
void orc_score(const uint16_t* q, const double* w_head, int heads, int dim,
               const uint16_t* keys, int64_t nblk, double* out, int nthreads) {
  std::vector<double> qd(static_cast<size_t>(heads) * dim);
  for (size_t i = 0; i < qd.size(); ++i) qd[i] = bf16_to_f64(q[i]);
  auto work = [&](int64_t b0, int64_t b1) {
    std::vector<double> kd(dim);
    for (int64_t b = b0; b < b1; ++b) {
      for (int d = 0; d < dim; ++d) kd[d] = bf16_to_f64(keys[b * dim + d]);
      double s = 0.0;
      for (int h = 0; h < heads; ++h) {
        double dot = 0.0;
        for (int d = 0; d < dim; ++d) dot += qd[h * dim + d] * kd[d];
        s += w_head[h] * (dot > 0.0 ? dot : 0.0);
      }
      out[b] = s;
    }
  };
  const int nt = pick_threads(nthreads);
  if (nt <= 1 || nblk < 4096) {
    work(0, nblk);
    return;
  }
  std::vector<std::thread> pool;
  for (int t = 0; t < nt; ++t) {
    int64_t b0 = nblk * t / nt, b1 = nblk * (t + 1) / nt;
    pool.emplace_back(work, b0, b1);
  }
  for (auto& th : pool) th.join();
}

// ---- INT8 pooled-key cache --------------------------------------------------
// [W1] section "양자화: W8A8와 혼합 캐시": the indexer's far, compressed cache
// entries are kept in INT8.  The page gives no scale convention; the reading
// followed here: a vector x (one pooled block, or one query head) is stored
// as symmetric codes c_i = round-half-even(x_i / 2^e) with one power-of-two
// scale 2^e, e the smallest integer with max_i |x_i| <= 127 * 2^e (so every
// |c_i| <= 127), e not below -149 (the smallest fp32 power of two); an
// all-zero vector takes e = 0.

// Returns e and writes the n codes.  The exponent is found by walking down
// from one that satisfies the bound (amax < 2^(ilogb(amax) + 1)) until one
// step further would break it.
int orc_quant_i8(const double* x, int n, int8_t* codes) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(x[i]));
  int e = 0;
  if (amax > 0.0) {
    e = std::ilogb(amax) + 1;
    while (e > -149 && amax <= 127.0 * std::ldexp(1.0, e - 1)) --e;
  }
  for (int i = 0; i < n; ++i) {
    const double c = std::nearbyint(std::ldexp(x[i], -e));  // exact scaling, then RNE
    codes[i] = static_cast<int8_t>(c);
  }
  return e;
}

// IndexPool write into the INT8 cache: the exact pooled sum of each complete
// block (as orc_pool, before any bf16 rounding) quantised per block; scale[b]
// receives 2^e of block b.
void orc_pool_i8(const uint16_t* raw, int64_t n_tok, int dim, int pool, const double* w,
                 int8_t* codes, double* scale) {
  const int64_t nblk = n_tok / pool;
  std::vector<double> acc(dim);
  for (int64_t b = 0; b < nblk; ++b) {
    for (int d = 0; d < dim; ++d) {
      double s = 0.0;
      for (int i = 0; i < pool; ++i) s += w[i] * bf16_to_f64(raw[(b * pool + i) * dim + d]);
      acc[d] = s;
    }
    scale[b] = std::ldexp(1.0, orc_quant_i8(acc.data(), dim, codes + b * dim));
  }
}

// Indexer score against the INT8 cache: every query head h is quantised the
// same way (codes qc_h, scale 2^{e_h}); then
//   s[b] = scale[b] * sum_h w_h 2^{e_h} max(0, sum_d qc_h[d] * kc_b[d]),
// i.e. the score of the dequantised query against the dequantised key.
void orc_score_i8(const uint16_t* q, const double* w_head, int heads, int dim,
                  const int8_t* codes, const double* scale, int64_t nblk, double* out,
                  int nthreads) {
  std::vector<int8_t> qc(static_cast<size_t>(heads) * dim);
  std::vector<double> qs(heads), row(dim);
  for (int h = 0; h < heads; ++h) {
    for (int d = 0; d < dim; ++d) row[d] = bf16_to_f64(q[h * dim + d]);
    qs[h] = std::ldexp(1.0, orc_quant_i8(row.data(), dim, qc.data() + h * dim));
  }
  auto work = [&](int64_t b0, int64_t b1) {
    for (int64_t b = b0; b < b1; ++b) {
      double s = 0.0;
      for (int h = 0; h < heads; ++h) {
        double dot = 0.0;
        for (int d = 0; d < dim; ++d)
          dot += static_cast<double>(qc[h * dim + d]) * static_cast<double>(codes[b * dim + d]);
        s += w_head[h] * qs[h] * (dot > 0.0 ? dot : 0.0);
      }
      out[b] = scale[b] * s;
    }
  };
  const int nt = pick_threads(nthreads);
  if (nt <= 1 || nblk < 4096) {
    work(0, nblk);
    return;
  }
  std::vector<std::thread> pool;
  for (int t = 0; t < nt; ++t) {
    int64_t b0 = nblk * t / nt, b1 = nblk * (t + 1) / nt;
    pool.emplace_back(work, b0, b1);
  }
  for (auto& th : pool) th.join();
}

// ---- FP8 (E4M3) latent cache -------------------------------------------------
// [W1] section "양자화: W8A8와 혼합 캐시": recent, important cache entries are
// kept in FP8.  Reading followed here for the MLA latent rows: a row x is
// stored as E4M3 codes (4 exponent bits with bias 7, 3 mantissa bits,
// largest finite value 448, subnormal step 2^-9) of x / 2^e, one
// power-of-two scale 2^e per row, e the smallest integer with
// max |x| <= 448 * 2^e (not below -149; 0 for an all-zero row), rounding to
// nearest with ties to even.

// Nearest-even E4M3 value of v, |v| <= 448: keep 4 significant bits, the
// subnormal step 2^-9 being the finest.
static double e4m3_round(double v) {
  if (v == 0.0) return v;
  int E = 0;
  std::frexp(std::fabs(v), &E);  // |v| = m 2^E, m in [0.5, 1)
  int qe = E - 4;                // weight of the last kept bit
  if (qe < -9) qe = -9;
  const double r = std::ldexp(std::nearbyint(std::ldexp(std::fabs(v), -qe)), qe);
  return std::signbit(v) ? -r : r;
}

// Bit pattern of an E4M3 value r (one that e4m3_round returns).
uint8_t orc_e4m3_bits(double v) {
  const double r = e4m3_round(v);
  const uint8_t sign = std::signbit(r) ? 0x80 : 0x00;
  const double a = std::fabs(r);
  if (a == 0.0) return sign;
  if (a < std::ldexp(1.0, -6))  // subnormal: a = mant * 2^-9
    return sign | static_cast<uint8_t>(std::ldexp(a, 9));
  int E = 0;
  std::frexp(a, &E);  // a = 1.f * 2^(E-1)
  const int mant = static_cast<int>(std::ldexp(a, 4 - E)) - 8;  // 3 fraction bits
  return sign | static_cast<uint8_t>(((E - 1 + 7) << 3) | mant);
}

// Value of an E4M3 bit pattern (finite patterns only).
double orc_e4m3_value(uint8_t bits) {
  const int ex = (bits >> 3) & 15, mant = bits & 7;
  const double a = ex == 0 ? std::ldexp(mant, -9) : std::ldexp(8 + mant, ex - 7 - 3);
  return (bits & 0x80) ? -a : a;
}

// Returns e and writes the n E4M3 codes of x / 2^e.
int orc_quant_e4m3(const double* x, int n, uint8_t* codes) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(x[i]));
  int e = 0;
  if (amax > 0.0) {
    e = std::ilogb(amax) + 1;  // amax < 2^e <= 448 * 2^e
    while (e > -149 && amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;
  }
  for (int i = 0; i < n; ++i) codes[i] = orc_e4m3_bits(std::ldexp(x[i], -e));
  return e;
}

// Top-k block selection [W4 "수렴점 2": keep the 512 highest-scoring 4-token
// blocks]: full sort on (score descending, block ascending) -- equal scores
// go to the lower block index -- keep the first min(K, nblk), return them
// in ascending block order.  Scores are compared after rounding to fp32;
// -0 and +0 compare equal.
int64_t orc_topk(const double* s, int64_t nblk, int64_t K, int32_t* idx_out) {
  std::vector<std::pair<float, int64_t>> v(static_cast<size_t>(nblk));
  for (int64_t b = 0; b < nblk; ++b) v[b] = {static_cast<float>(s[b]), b};
  std::sort(v.begin(), v.end(), [](const auto& a, const auto& c) {
    if (a.first != c.first) return a.first > c.first;
    return a.second < c.second;
  });
  const int64_t k = std::min(K, nblk);
  std::vector<int64_t> sel(static_cast<size_t>(k));
  for (int64_t i = 0; i < k; ++i) sel[i] = v[i].second;
  std::sort(sel.begin(), sel.end());
  for (int64_t i = 0; i < k; ++i) idx_out[i] = static_cast<int32_t>(sel[i]);
  return k;
}

// Positions attended by a query that sees n_vis tokens: the 4 tokens of
// every selected block, then the partial tail n_vis - n_vis % pool .. n_vis-1
// (those tokens have no pooled key yet, so they are always kept).
int64_t orc_token_set(const int32_t* idx, int64_t count, int64_t n_vis,
                      int pool, int64_t* pos_out) {
  int64_t m = 0;
  for (int64_t j = 0; j < count; ++j)
    for (int i = 0; i < pool; ++i) pos_out[m++] = static_cast<int64_t>(idx[j]) * pool + i;
  for (int64_t t = (n_vis / pool) * pool; t < n_vis; ++t) pos_out[m++] = t;
  return m;
}

// Softmax attention of every head over the gathered latent rows
// [W3 "실제로 바꾸는 것": MLA runs on the selected positions only].
// Absorbed MLA with NoPE [W4 "위치 인코딩"]: the latent row c_t is both key and
// value, shared by all heads:
//   z_t = sm_scale * q_h . c_t,  o_h = sum_t softmax(z)_t c_t,
//   lse_h = log sum_t exp(z_t).
void orc_attention(const uint16_t* q, int heads, int dim, const uint16_t* rows,
                   int64_t S, double sm_scale, double* out, double* lse) {
  if (S <= 0) {  // a query that sees no token: zero output, lse = -inf
    for (int64_t i = 0; i < static_cast<int64_t>(heads) * dim; ++i) out[i] = 0.0;
    if (lse)
      for (int h = 0; h < heads; ++h) lse[h] = -INFINITY;
    return;
  }
  std::vector<double> c(static_cast<size_t>(S) * dim);
  for (size_t i = 0; i < c.size(); ++i) c[i] = bf16_to_f64(rows[i]);
  std::vector<double> z(static_cast<size_t>(S));
  for (int h = 0; h < heads; ++h) {
    std::vector<double> qh(dim);
    for (int d = 0; d < dim; ++d) qh[d] = bf16_to_f64(q[h * dim + d]);
    double m = -INFINITY;
    for (int64_t t = 0; t < S; ++t) {
      double dot = 0.0;
      for (int d = 0; d < dim; ++d) dot += qh[d] * c[t * dim + d];
      z[t] = sm_scale * dot;
      m = std::max(m, z[t]);
    }
    double l = 0.0;
    for (int64_t t = 0; t < S; ++t) {
      z[t] = std::exp(z[t] - m);
      l += z[t];
    }
    for (int d = 0; d < dim; ++d) {
      double acc = 0.0;
      for (int64_t t = 0; t < S; ++t) acc += z[t] * c[t * dim + d];
      out[h * dim + d] = acc / l;
    }
    if (lse) lse[h] = m + std::log(l);
  }
}

}  // extern "C"
