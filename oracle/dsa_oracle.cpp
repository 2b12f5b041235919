// DSA oracle — TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, CPU restatement of what DeepSeek Sparse Attention computes,
// written from the DeepSeek Sparse Attention page (kwkr.cn/news/60693):
//   * section 3.2 (lightning indexer): scores = relu(matmul(q, k^T) * scale),
//     scale = dim^-0.5;
//   * section 3.3 (fine-grained token selection): each query keeps its top-k
//     keys, then ordinary ("standard") softmax attention runs over only those;
//   * section 4.1 (precision): FP8 index stage, BF16 attention stage;
//   * section 4.2 (memory): all query heads share one K/V (MQA).
// Readings where the page is silent: causal keys s <= t (diagonal included);
// ties in score go to the lower key index; a row keeps all t+1 keys when
// t+1 <= k and pads indices with -1; indices are listed in (score desc, index
// asc) order; the attention softmax scale is D^-0.5.
//
// Only the tests, the package's smoke check and the benchmark's CPU-baseline
// leg may load this library.  It shares no code with the CUDA path.
//
// Arithmetic: every dot product is accumulated in double.  For FP8 E4M3
// inputs a double sum of d <= 256 products is exact (products have 8
// significant bits and span < 2^36 in magnitude); for BF16 inputs it is exact
// whenever the inputs are integers, as in every workload here.  The indexer
// score is then fp32(fp32(dot) * fp32(scale)), a single round-to-nearest
// product, and ReLU maps every non-positive score (and -0) to +0.  Attention
// logits, softmax and the weighted sum are double; the output is rounded once
// to BF16, nearest-even.
//
// Parity status: pinned (see tests/test_oracle.py for the pins: closed forms,
// library sorts and matmuls, torch SDPA for the dense limit, brute force).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---- number formats -------------------------------------------------------

// FP8 E4M3 (OCP 8-bit floating point, "E4M3" variant): 1 sign, 4 exponent
// (bias 7), 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); the only
// NaN encodings are S.1111.111; there are no infinities.
double fp8_e4m3_value(uint8_t b) {
  const int s = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
  if (e == 0xF && m == 7) return std::nan("");
  double v = (e == 0) ? std::ldexp(static_cast<double>(m), -9)
                      : std::ldexp(8.0 + m, e - 10);  // (1 + m/8) * 2^(e-7)
  return s ? -v : v;
}

// BF16: the upper 16 bits of an IEEE-754 binary32.
double bf16_value(uint16_t h) {
  const uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// Round a double to BF16 once, nearest-even (8 significant bits, exponent
// range of binary32, subnormal unit 2^-133).
uint16_t bf16_round(double x) {
  if (std::isnan(x)) return 0x7FC0;
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  const double a = std::fabs(x);
  if (a == 0.0) return sign;
  if (std::isinf(a)) return sign | 0x7F80;
  int e;
  std::frexp(a, &e);  // a = f * 2^e, f in [0.5, 1)
  int E = e - 1;      // a = 1.xxx * 2^E
  if (E < -126) {     // subnormal range: multiples of 2^-133
    const double q = std::nearbyint(std::ldexp(a, 133));  // default mode: ties to even
    return sign | static_cast<uint16_t>(q);  // q == 128 lands on the smallest normal
  }
  double q = std::nearbyint(std::ldexp(a, 7 - E));  // in [128, 256]
  if (q == 256.0) { q = 128.0; E += 1; }
  if (E > 127) return sign | 0x7F80;
  return sign | static_cast<uint16_t>(((E + 127) << 7) | (static_cast<int>(q) - 128));
}

// ---- decoded views --------------------------------------------------------

enum { IDX_FP8_E4M3 = 0, IDX_BF16 = 1 };

std::vector<double> decode_index(const void* p, int dtype, int64_t n) {
  std::vector<double> out(static_cast<size_t>(n));
  if (dtype == IDX_FP8_E4M3) {
    const uint8_t* b = static_cast<const uint8_t*>(p);
    for (int64_t i = 0; i < n; ++i) out[i] = fp8_e4m3_value(b[i]);
  } else {
    const uint16_t* h = static_cast<const uint16_t*>(p);
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_value(h[i]);
  }
  return out;
}

std::vector<double> decode_bf16(const uint16_t* p, int64_t n) {
  std::vector<double> out(static_cast<size_t>(n));
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_value(p[i]);
  return out;
}

// ---- the three steps ------------------------------------------------------

// Step 1, lightning indexer score of one (query, key) pair:
// relu(fp32(fp32(dot) * fp32(scale))), non-positive -> +0.
float index_score(const double* q, const double* k, int d, float scale) {
  double dot = 0.0;
  for (int j = 0; j < d; ++j) dot += q[j] * k[j];
  volatile float dotf = static_cast<float>(dot);
  volatile float sc = dotf * scale;  // one binary32 multiply, round-to-nearest
  return sc > 0.0f ? static_cast<float>(sc) : 0.0f;
}

// Step 2, selection: order keys 0..n-1 by (score desc, index asc), keep the
// first min(k, n), pad with -1 to length k.
void select_top_k(const std::vector<float>& score, int64_t n, int k, int32_t* out) {
  std::vector<int64_t> order(static_cast<size_t>(n));
  std::iota(order.begin(), order.end(), 0);
  auto before = [&](int64_t a, int64_t b) {
    if (score[a] != score[b]) return score[a] > score[b];
    return a < b;
  };
  const int64_t m = std::min<int64_t>(k, n);
  if (m < n) std::nth_element(order.begin(), order.begin() + m, order.end(), before);
  std::sort(order.begin(), order.begin() + m, before);
  for (int64_t i = 0; i < k; ++i) out[i] = (i < m) ? static_cast<int32_t>(order[i]) : -1;
}

// Step 3, softmax attention of H heads over the selected keys of one query.
void attend(const double* q /*[H, D]*/, const double* K, const double* V, const int32_t* sel,
            int k, int H, int D, double scale, uint16_t* out /*[H, D]*/) {
  std::vector<double> logit(static_cast<size_t>(k)), acc(static_cast<size_t>(D));
  for (int h = 0; h < H; ++h) {
    const double* qh = q + static_cast<int64_t>(h) * D;
    double mx = -INFINITY;
    int n = 0;
    for (int i = 0; i < k && sel[i] >= 0; ++i, ++n) {
      const double* kr = K + static_cast<int64_t>(sel[i]) * D;
      double dot = 0.0;
      for (int j = 0; j < D; ++j) dot += qh[j] * kr[j];
      logit[i] = dot * scale;
      mx = std::max(mx, logit[i]);
    }
    std::fill(acc.begin(), acc.end(), 0.0);
    double denom = 0.0;
    for (int i = 0; i < n; ++i) {
      const double p = std::exp(logit[i] - mx);
      denom += p;
      const double* vr = V + static_cast<int64_t>(sel[i]) * D;
      for (int j = 0; j < D; ++j) acc[j] += p * vr[j];
    }
    for (int j = 0; j < D; ++j)
      out[static_cast<int64_t>(h) * D + j] = bf16_round(n ? acc[j] / denom : 0.0);
  }
}

int set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) return nthreads;
  return omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

}  // namespace

extern "C" {

// Library versions of the format helpers, so tests can pin them against the
// OCP FP8 table, IEEE-754 and torch's conversions.
double oracle_fp8_e4m3_value(uint8_t b) { return fp8_e4m3_value(b); }
double oracle_bf16_value(uint16_t h) { return bf16_value(h); }
uint16_t oracle_bf16_round(double x) { return bf16_round(x); }

// Dense lightning-indexer scores, no mask: out[t, s] = relu(fp32(q_t.k_s) *
// scale) for t < Lq, s < Lk.  out is [Lq, Lk] float32.
void oracle_indexer_scores(const void* q_idx, const void* k_idx, int idx_dtype, int d,
                           float scale, int64_t Lq, int64_t Lk, float* out, int nthreads) {
  const std::vector<double> q = decode_index(q_idx, idx_dtype, Lq * d);
  const std::vector<double> k = decode_index(k_idx, idx_dtype, Lk * d);
  const int nt = set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16) num_threads(nt)
  for (int64_t t = 0; t < Lq; ++t)
    for (int64_t s = 0; s < Lk; ++s)
      out[t * Lk + s] = index_score(&q[t * d], &k[s * d], d, scale);
}

// Prefill of one causal sequence, evaluated for the listed query rows only.
// Inputs: q_idx, k_idx [L, d] (FP8 E4M3 bytes or BF16 bits), Q [L, H, D],
// K, V [L, D] (BF16 bits).  Outputs for row list entry i (query t = rows[i]):
// indices[i, 0:top_k] and O[i, H, D] (BF16 bits).  Either output may be null.
void oracle_prefill_rows(const void* q_idx, const void* k_idx, int idx_dtype, int d,
                         float idx_scale, const uint16_t* Q, const uint16_t* K,
                         const uint16_t* V, int64_t L, int H, int D, double attn_scale,
                         int top_k, const int64_t* rows, int64_t nrows, int32_t* indices,
                         uint16_t* O, int nthreads) {
  const std::vector<double> qv = decode_index(q_idx, idx_dtype, L * d);
  const std::vector<double> kv = decode_index(k_idx, idx_dtype, L * d);
  std::vector<double> Kd, Vd;
  if (O) {
    Kd = decode_bf16(K, L * D);
    Vd = decode_bf16(V, L * D);
  }
  const int nt = set_threads(nthreads);
#pragma omp parallel num_threads(nt)
  {
    std::vector<float> score;
    std::vector<int32_t> sel(static_cast<size_t>(top_k));
    std::vector<double> qh(static_cast<size_t>(H) * D);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
      const int64_t t = rows[i];
      score.assign(static_cast<size_t>(t + 1), 0.0f);
      for (int64_t s = 0; s <= t; ++s)
        score[s] = index_score(&qv[t * d], &kv[s * d], d, idx_scale);
      select_top_k(score, t + 1, top_k, sel.data());
      if (indices) std::memcpy(indices + i * top_k, sel.data(), sizeof(int32_t) * top_k);
      if (O) {
        for (int64_t j = 0; j < static_cast<int64_t>(H) * D; ++j)
          qh[j] = bf16_value(Q[t * H * D + j]);
        attend(qh.data(), Kd.data(), Vd.data(), sel.data(), top_k, H, D, attn_scale,
               O + i * H * D);
      }
    }
  }
}

// Batched decode: sequence b owns cache rows seq_start[b] .. seq_start[b+1]-1
// of k_idx [*, d], K, V [*, D]; its one new query (q_idx[b], Q[b]) sits at
// position len_b - 1 and sees all len_b rows.  Outputs indices [B, top_k]
// (may be null) and O [B, H, D].
void oracle_decode(const void* k_idx, const uint16_t* K, const uint16_t* V,
                   const int64_t* seq_start, int B, int idx_dtype, int d, int D,
                   const void* q_idx, const uint16_t* Q, int H, int top_k, float idx_scale,
                   double attn_scale, int32_t* indices, uint16_t* O, int nthreads) {
  const int esize = (idx_dtype == IDX_FP8_E4M3) ? 1 : 2;
  const int nt = set_threads(nthreads);
#pragma omp parallel num_threads(nt)
  {
    std::vector<float> score;
    std::vector<int32_t> sel(static_cast<size_t>(top_k));
#pragma omp for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
      const int64_t r0 = seq_start[b], n = seq_start[b + 1] - seq_start[b];
      const std::vector<double> kv = decode_index(
          static_cast<const uint8_t*>(k_idx) + r0 * d * esize, idx_dtype, n * d);
      const std::vector<double> qv = decode_index(
          static_cast<const uint8_t*>(q_idx) + static_cast<int64_t>(b) * d * esize, idx_dtype, d);
      score.assign(static_cast<size_t>(n), 0.0f);
      for (int64_t s = 0; s < n; ++s) score[s] = index_score(qv.data(), &kv[s * d], d, idx_scale);
      select_top_k(score, n, top_k, sel.data());
      if (indices) std::memcpy(indices + static_cast<int64_t>(b) * top_k, sel.data(),
                               sizeof(int32_t) * top_k);
      if (O) {
        // Decode only the selected rows' K/V.
        std::vector<double> Ks(static_cast<size_t>(top_k) * D), Vs(static_cast<size_t>(top_k) * D);
        std::vector<int32_t> local(static_cast<size_t>(top_k));
        for (int i = 0; i < top_k; ++i) {
          local[i] = sel[i] >= 0 ? i : -1;
          if (sel[i] < 0) continue;
          for (int j = 0; j < D; ++j) {
            Ks[static_cast<int64_t>(i) * D + j] = bf16_value(K[(r0 + sel[i]) * D + j]);
            Vs[static_cast<int64_t>(i) * D + j] = bf16_value(V[(r0 + sel[i]) * D + j]);
          }
        }
        std::vector<double> qh(static_cast<size_t>(H) * D);
        for (int64_t j = 0; j < static_cast<int64_t>(H) * D; ++j)
          qh[j] = bf16_value(Q[static_cast<int64_t>(b) * H * D + j]);
        attend(qh.data(), Ks.data(), Vs.data(), local.data(), top_k, H, D, attn_scale,
               O + static_cast<int64_t>(b) * H * D);
      }
    }
  }
}

int oracle_max_threads(void) { return set_threads(0); }

}  // extern "C"
