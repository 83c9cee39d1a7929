// Plain CPU oracle of the hybrid compressed attention path, in C++17 and
// float64, parallel over query rows (OpenMP).
//
// TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
// CPU-baseline legs of the benchmark load this library (through
// oracle/cpp_oracle.py). It shares no code, header, table or helper with the
// CUDA library, and neither side includes or links the other.
//
// It restates, step by step, what the float64 numpy oracle (cslc_oracle.py)
// computes, from the same passages of the source pages:
//   "从论文出发，逐层剖析 CSA / HCA 混注意力、mHC 残差连接与 Muon 优化器": §1.1 CSA and its
//     工程细节 paragraph (m = 4, top-k = 1024, overlapped C^a / C^b windows of 2m
//     tokens), §1.2 HCA (m' = 128, dense), §1.4 存储格式混 (RoPE dims BF16, the
//     other dims FP8).
//   "读完这篇你就搞懂 DeepSeek v4 了": §三 压缩机制 (per-dimension weighting of the
//     tokens of a group, two consecutive groups joined, 4 W + 2 B), 闪电索引
//     (score every entry per query, weight per head, top-k), 注意力计算 (ordinary
//     attention over the selected entries, KV shared), HCA 步骤简化.
// Readings where the pages leave a step open are the numpy oracle's R1-R8:
// softmax over the window of (z + positional bias) per channel weights c;
// entry i's window ends at token (i+1)m-1 and a query at position p sees entry
// i iff (i+1)m-1 <= p; scores S = sum_h w_h ReLU(q_h . k); top-k ties go to the
// smaller index and the set is returned ascending, -1 padded; K = V = entry;
// FP8 e4m3 with one fp32 scale per entry (amax / 448, 1 when amax = 0).
//
// Inputs are float64 arrays holding the tensors' exact values (bf16 inputs
// convert to double exactly). All arithmetic is float64; results are rounded
// only at the path's storage points: entries and outputs to bf16 (round to
// nearest, ties to even), scores and lse to fp32, KV to e4m3 codes.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr double kInf = std::numeric_limits<double>::infinity();
constexpr double kBf16Max = (2.0 - 1.0 / 128.0) * 1.7014118346046923e38;   // (2 - 2^-7) * 2^127
constexpr double kE4m3Max = 448.0;

// Nearest bfloat16 value (8 significant bits, quantum 2^-133 below 2^-126),
// ties to even; values at or past the overflow midpoint become +-inf.
double round_bf16(double x) {
  if (!std::isfinite(x) || x == 0.0) return x;
  int e = 0;
  std::frexp(x, &e);   // x = f * 2^e, 0.5 <= |f| < 1
  const double quantum = std::ldexp(1.0, std::max(e, -125) - 8);
  const double r = std::nearbyint(x / quantum) * quantum;   // default rounding: to nearest, ties to even
  if (std::fabs(r) > kBf16Max) return std::copysign(kInf, r);
  return r;
}

double round_fp32(double x) { return static_cast<double>(static_cast<float>(x)); }

long long n_visible(long long p, long long m, long long n_c) {
  if (p < 0) return 0;
  return std::min(n_c, (p + 1) / m);
}

// Tokens, slots and C^b membership of compressed entry i.
int window(long long i, int m, bool overlap, long long* tokens, int* slots, bool* is_prev) {
  int n = 0;
  if (overlap && i > 0) {
    for (int s = 0; s < m; ++s) { tokens[n] = (i - 1) * m + s; slots[n] = s; is_prev[n] = true; ++n; }
  }
  for (int s = 0; s < m; ++s) {
    tokens[n] = i * m + s;
    slots[n] = overlap ? m + s : s;
    is_prev[n] = false;
    ++n;
  }
  return n;
}

// Softmax attention of H heads over n entries (K = V); o unrounded.
void attend(const double* q, const double* kv, int H, int D, long long n, double scale, double* o, double* lse) {
  if (n == 0) {
    std::fill(o, o + (size_t)H * D, 0.0);
    for (int h = 0; h < H; ++h) lse[h] = -kInf;
    return;
  }
  std::vector<double> logit(n), acc(D);
  for (int h = 0; h < H; ++h) {
    const double* qh = q + (size_t)h * D;
    double mx = -kInf;
    for (long long i = 0; i < n; ++i) {
      double d = 0.0;
      const double* ki = kv + (size_t)i * D;
      for (int c = 0; c < D; ++c) d += qh[c] * ki[c];
      logit[i] = scale * d;
      mx = std::max(mx, logit[i]);
    }
    double denom = 0.0;
    std::fill(acc.begin(), acc.end(), 0.0);
    for (long long i = 0; i < n; ++i) {
      const double p = std::exp(logit[i] - mx);
      denom += p;
      const double* ki = kv + (size_t)i * D;
      for (int c = 0; c < D; ++c) acc[c] += p * ki[c];
    }
    for (int c = 0; c < D; ++c) o[(size_t)h * D + c] = acc[c] / denom;
    lse[h] = mx + std::log(denom);
  }
}

// Order of the top-k: larger score first, ties to the smaller index; a NaN
// score ranks below every number.
bool ranks_before(double sa, long long a, double sb, long long b) {
  const bool na = std::isnan(sa), nb = std::isnan(sb);
  if (na != nb) return nb;
  if (!na && sa != sb) return sa > sb;
  return a < b;
}

void topk_row(const double* s, long long n_vis, int k, int32_t* out) {
  std::vector<long long> cand(n_vis);
  for (long long i = 0; i < n_vis; ++i) cand[i] = i;
  std::sort(cand.begin(), cand.end(), [&](long long a, long long b) { return ranks_before(s[a], a, s[b], b); });
  const long long kk = std::min<long long>(k, n_vis);
  std::sort(cand.begin(), cand.begin() + kk);
  for (int j = 0; j < k; ++j) out[j] = j < kk ? (int32_t)cand[j] : -1;
}

// E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
// subnormal (mantissa/8 * 2^-6); S.1111.111 is NaN; no infinities.
double e4m3_value(uint8_t code) {
  const double sign = (code & 0x80) ? -1.0 : 1.0;
  const int ex = (code >> 3) & 0xF, man = code & 0x7;
  if (ex == 0xF && man == 0x7) return std::numeric_limits<double>::quiet_NaN();
  if (ex == 0) return sign * (man / 8.0) * std::ldexp(1.0, -6);
  return sign * (1.0 + man / 8.0) * std::ldexp(1.0, ex - 7);
}

// Nearest E4M3 code, ties to even; finite values past the range saturate to 448.
uint8_t e4m3_code(double x) {
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  const double a = std::fabs(x);
  if (!(a > 0.0)) return sign;   // +-0 (NaN input is outside the method's domain)
  int e = 0;
  std::frexp(a, &e);
  const double quantum = std::ldexp(1.0, std::max(e, -5) - 4);   // 4 significant bits; 2^-9 below 2^-6
  const double r = std::min(std::nearbyint(a / quantum) * quantum, kE4m3Max);
  if (r == 0.0) return sign;
  if (r < std::ldexp(1.0, -6)) return sign | (uint8_t)std::nearbyint(r / std::ldexp(1.0, -9));
  int er = 0;
  std::frexp(r, &er);
  const int ef = er - 1 + 7;
  const int mf = (int)std::nearbyint((r / std::ldexp(1.0, er - 1) - 1.0) * 8.0);
  return sign | (uint8_t)(ef << 3) | (uint8_t)mf;
}

}  // namespace

extern "C" {

int orc_threads(void) {
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

void orc_round_bf16(const double* x, long long n, double* out) {
  for (long long i = 0; i < n; ++i) out[i] = round_bf16(x[i]);
}

void orc_round_fp32(const double* x, long long n, double* out) {
  for (long long i = 0; i < n; ++i) out[i] = round_fp32(x[i]);
}

long long orc_n_visible(long long p, long long m, long long n_c) { return n_visible(p, m, n_c); }

int orc_compression_window(long long i, int m, int overlap, long long* tokens, int* slots, unsigned char* is_prev) {
  bool tmp[256];   // a window holds at most 2m <= 256 tokens
  const int n = window(i, m, overlap != 0, tokens, slots, tmp);
  for (int j = 0; j < n; ++j) is_prev[j] = tmp[j] ? 1 : 0;
  return n;
}

// One learned projection of the compressor front end: out[r, n] = sum_k
// h[r, k] W[n, k] for the rows r of h [rows, d_model] and W [D, d_model].
void orc_project(const double* h, const double* W, long long rows, int d_model, int D, double* out) {
#pragma omp parallel for schedule(static)
  for (long long r = 0; r < rows; ++r)
    for (int n = 0; n < D; ++n) {
      double acc = 0.0;
      for (int k = 0; k < d_model; ++k) acc += h[(size_t)r * d_model + k] * W[(size_t)n * d_model + k];
      out[(size_t)r * D + n] = acc;
    }
}

// Per-channel softmax over the W window tokens of (z + bias[slot]).
// zw: [W, D]; bias_rows: [W, D]; out: [W, D].
void orc_compression_weights(const double* zw, const double* bias_rows, int W, int D, double* out) {
  for (int c = 0; c < D; ++c) {
    double mx = -kInf;
    for (int t = 0; t < W; ++t) mx = std::max(mx, zw[(size_t)t * D + c] + bias_rows[(size_t)t * D + c]);
    double den = 0.0;
    for (int t = 0; t < W; ++t) {
      const double e = std::exp(zw[(size_t)t * D + c] + bias_rows[(size_t)t * D + c] - mx);
      out[(size_t)t * D + c] = e;
      den += e;
    }
    for (int t = 0; t < W; ++t) out[(size_t)t * D + c] /= den;
  }
}

// Compressed entries out[b, i, :] for every complete window; c_b / z_b (or
// NULL) feed the C^b half of CSA windows.
void orc_compress(const double* c, const double* z, const double* bias, const double* c_b, const double* z_b,
                  int B, long long L, int D, int m, int overlap, int round_output, double* out) {
  const long long n_c = L / m;
  const double* cb = c_b ? c_b : c;
  const double* zb = z_b ? z_b : z;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b) {
    for (long long i = 0; i < n_c; ++i) {
      long long tokens[256];
      int slots[256];
      bool prev[256];
      const int W = window(i, m, overlap != 0, tokens, slots, prev);
      std::vector<double> zw((size_t)W * D), bw((size_t)W * D), wt((size_t)W * D);
      for (int t = 0; t < W; ++t) {
        const double* zs = (prev[t] ? zb : z) + ((size_t)b * L + tokens[t]) * D;
        for (int ch = 0; ch < D; ++ch) {
          zw[(size_t)t * D + ch] = zs[ch];
          bw[(size_t)t * D + ch] = bias[(size_t)slots[t] * D + ch];
        }
      }
      orc_compression_weights(zw.data(), bw.data(), W, D, wt.data());
      double* o = out + ((size_t)b * n_c + i) * D;
      for (int ch = 0; ch < D; ++ch) {
        double acc = 0.0;
        for (int t = 0; t < W; ++t) {
          const double* cs = (prev[t] ? cb : c) + ((size_t)b * L + tokens[t]) * D;
          acc += wt[(size_t)t * D + ch] * cs[ch];
        }
        o[ch] = round_output ? round_bf16(acc) : acc;
      }
    }
  }
}

// Indexer scores of the requested query rows (row t is absolute position
// q_pos0 + t); entries past n_vis are -inf; fp32-rounded. out: [B, n_rows, Nc].
// With `compact`, q_idx and w hold only the requested rows ([B, n_rows, ...]).
void orc_indexer_scores(const double* q_idx, const double* w, const double* k_idx, int B, long long L, int HI, int dI,
                        long long Nc, int m, long long q_pos0, const long long* rows, long long n_rows, int compact,
                        double* out) {
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
  for (int b = 0; b < B; ++b) {
    for (long long r = 0; r < n_rows; ++r) {
      const long long t = rows ? rows[r] : r;
      const long long nv = n_visible(q_pos0 + t, m, Nc);
      double* o = out + ((size_t)b * n_rows + r) * Nc;
      const long long src = compact ? r : t;
      const long long rows_in = compact ? n_rows : L;
      const double* qt = q_idx + ((size_t)b * rows_in + src) * HI * dI;
      const double* wt = w + ((size_t)b * rows_in + src) * HI;
      for (long long i = 0; i < Nc; ++i) {
        if (i >= nv) { o[i] = -kInf; continue; }
        const double* ki = k_idx + ((size_t)b * Nc + i) * dI;
        double s = 0.0;
        for (int h = 0; h < HI; ++h) {
          double d = 0.0;
          for (int c = 0; c < dI; ++c) d += qt[(size_t)h * dI + c] * ki[c];
          s += wt[h] * std::max(d, 0.0);
        }
        o[i] = round_fp32(s);
      }
    }
  }
}

void orc_topk_select_row(const double* s, long long n_vis, int k, int32_t* out) { topk_row(s, n_vis, k, out); }

// Top-k rows of a score tensor [B, R, Nc]; row r is query row rows[r] (or r).
void orc_topk_select(const double* scores, int B, long long R, long long Nc, int m, int k, long long q_pos0,
                     const long long* rows, int32_t* out) {
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
  for (int b = 0; b < B; ++b)
    for (long long r = 0; r < R; ++r) {
      const long long t = rows ? rows[r] : r;
      topk_row(scores + ((size_t)b * R + r) * Nc, n_visible(q_pos0 + t, m, Nc), k, out + ((size_t)b * R + r) * k);
    }
}

void orc_attend(const double* q, const double* kv, int H, int D, long long n, double scale, double* o, double* lse) {
  attend(q, kv, H, D, n, scale, o, lse);
}

// CSA core attention over the selected entries (-1 = empty slot) of the
// requested rows; o bf16-rounded [B, n_rows, H, D], lse fp32 [B, n_rows, H].
void orc_sparse_attention(const double* q, const double* e, const int32_t* idx, int B, long long L, int H, int D,
                          long long Nc, int k, double scale, const long long* rows, long long n_rows, double* o,
                          double* lse) {
#pragma omp parallel for collapse(2) schedule(dynamic, 2)
  for (int b = 0; b < B; ++b) {
    for (long long r = 0; r < n_rows; ++r) {
      const long long t = rows ? rows[r] : r;
      const int32_t* sel = idx + ((size_t)b * L + t) * k;
      std::vector<double> kv;
      kv.reserve((size_t)k * D);
      long long n = 0;
      for (int j = 0; j < k; ++j) {
        if (sel[j] < 0) continue;
        const double* ei = e + ((size_t)b * Nc + sel[j]) * D;
        kv.insert(kv.end(), ei, ei + D);
        ++n;
      }
      double* ob = o + ((size_t)b * n_rows + r) * H * D;
      double* lb = lse + ((size_t)b * n_rows + r) * H;
      attend(q + ((size_t)b * L + t) * H * D, kv.data(), H, D, n, scale, ob, lb);
      for (long long x = 0; x < (long long)H * D; ++x) ob[x] = round_bf16(ob[x]);
      for (int h = 0; h < H; ++h) lb[h] = round_fp32(lb[h]);
    }
  }
}

// HCA core attention: dense over the visible entries of the requested rows.
// With `compact`, q holds only the requested rows ([B, n_rows, H, D]).
void orc_dense_causal_attention(const double* q, const double* e, int B, long long L, int H, int D, long long Nc,
                                int m, double scale, long long q_pos0, const long long* rows, long long n_rows,
                                int compact, double* o, double* lse) {
#pragma omp parallel for collapse(2) schedule(dynamic, 2)
  for (int b = 0; b < B; ++b) {
    for (long long r = 0; r < n_rows; ++r) {
      const long long t = rows ? rows[r] : r;
      double* ob = o + ((size_t)b * n_rows + r) * H * D;
      double* lb = lse + ((size_t)b * n_rows + r) * H;
      const double* qt = compact ? q + ((size_t)b * n_rows + r) * H * D : q + ((size_t)b * L + t) * H * D;
      attend(qt, e + (size_t)b * Nc * D, H, D, n_visible(q_pos0 + t, m, Nc), scale, ob, lb);
      for (long long x = 0; x < (long long)H * D; ++x) ob[x] = round_bf16(ob[x]);
      for (int h = 0; h < H; ++h) lb[h] = round_fp32(lb[h]);
    }
  }
}

void orc_e4m3_decode(const uint8_t* codes, long long n, double* out) {
  for (long long i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
}

void orc_e4m3_encode(const double* x, long long n, uint8_t* out) {
  for (long long i = 0; i < n; ++i) out[i] = e4m3_code(x[i]);
}

// Mixed decode layout of n_entries entries [n, 128]: codes of dims 0..63
// divided by the entry scale (computed in fp32), dims 64..127 unchanged, scale.
void orc_quantize_kv_mixed(const double* e, long long n, uint8_t* codes, double* rope, float* scale) {
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < n; ++i) {
    const double* ei = e + (size_t)i * 128;
    float amax = 0.f;
    for (int c = 0; c < 64; ++c) amax = std::max(amax, std::fabs((float)ei[c]));
    const float s = amax > 0.f ? amax / (float)kE4m3Max : 1.0f;
    scale[i] = s;
    for (int c = 0; c < 64; ++c) codes[(size_t)i * 64 + c] = e4m3_code((double)((float)ei[c] / s));
    for (int c = 0; c < 64; ++c) rope[(size_t)i * 64 + c] = ei[64 + c];
  }
}

void orc_dequantize_kv_mixed(const uint8_t* codes, const double* rope, const float* scale, long long n, double* out) {
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < n; ++i) {
    for (int c = 0; c < 64; ++c) out[(size_t)i * 128 + c] = e4m3_value(codes[(size_t)i * 64 + c]) * (double)scale[i];
    for (int c = 0; c < 64; ++c) out[(size_t)i * 128 + 64 + c] = rope[(size_t)i * 64 + c];
  }
}

// Indexer scores of one query per sequence over its n_entries[b] entries
// ([B, N], -inf past n_entries[b], fp32-rounded).
void orc_decode_indexer_scores(const double* q_idx, const double* w, const double* k_idx, const long long* n_entries,
                               int B, long long N, int HI, int dI, double* out) {
  for (int b = 0; b < B; ++b) {
    const long long n = n_entries[b];
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < N; ++i) {
      if (i >= n) { out[(size_t)b * N + i] = -kInf; continue; }
      const double* ki = k_idx + ((size_t)b * N + i) * dI;
      double s = 0.0;
      for (int h = 0; h < HI; ++h) {
        double d = 0.0;
        for (int c = 0; c < dI; ++c) d += q_idx[((size_t)b * HI + h) * dI + c] * ki[c];
        s += w[(size_t)b * HI + h] * std::max(d, 0.0);
      }
      out[(size_t)b * N + i] = round_fp32(s);
    }
  }
}

// One CSA decode layer: top-k of the scores (given, or the indexer's), then
// attention over kv_hat [B, N, 128]. o bf16-rounded [B, H, D]; idx [B, topk].
void orc_decode_csa_layer(const double* q, const double* scores, const double* kv_hat, const long long* n_entries,
                          int B, int H, int D, long long N, int topk, double scale, double* o, int32_t* idx) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int b = 0; b < B; ++b) {
    int32_t* sel = idx + (size_t)b * topk;
    topk_row(scores + (size_t)b * N, n_entries[b], topk, sel);
    std::vector<double> kv;
    long long n = 0;
    for (int j = 0; j < topk; ++j) {
      if (sel[j] < 0) continue;
      const double* ei = kv_hat + ((size_t)b * N + sel[j]) * D;
      kv.insert(kv.end(), ei, ei + D);
      ++n;
    }
    std::vector<double> lse(H);
    double* ob = o + (size_t)b * H * D;
    attend(q + (size_t)b * H * D, kv.data(), H, D, n, scale, ob, lse.data());
    for (long long x = 0; x < (long long)H * D; ++x) ob[x] = round_bf16(ob[x]);
  }
}

// One HCA decode layer: dense attention over all n_entries[b] entries.
void orc_decode_hca_layer(const double* q, const double* kv_hat, const long long* n_entries, int B, int H, int D,
                          long long N, double scale, double* o) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int b = 0; b < B; ++b) {
    std::vector<double> lse(H);
    double* ob = o + (size_t)b * H * D;
    attend(q + (size_t)b * H * D, kv_hat + (size_t)b * N * D, H, D, n_entries[b], scale, ob, lse.data());
    for (long long x = 0; x < (long long)H * D; ++x) ob[x] = round_bf16(ob[x]);
  }
}

}  // extern "C"
