// hca_oracle_c.cpp -- plain, slow C++ oracle of DeepSeek-V4 hybrid compressed
// attention (CSA + HCA), in double precision.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path calls or links this
// file; only tests/, __graft_entry__.smoke() and bench.py's CPU baseline and
// reference arm load it (through oracle/hca_oracle_c.py).  It shares no code
// with the CUDA path or with oracle/hca_oracle.py: it is a second, independent
// restatement of the same steps, as straight loops:
//
//   [J]  juejin.cn "DeepSeek-V4 技术报告简要解读": §2.3.1 (CSA) Eq.(11)-(12)
//        block compression, Eq.(16) index score, Eq.(17) top-k, Eq.(18)-(19)
//        shared-KV MQA; §2.3.2 (HCA) Eq.(22)-(23); §2.3.3 partial RoPE,
//        sliding window, attention sink Eq.(27).
//   [Z]  1zeryu.github.io "DeepSeek-V4：算法架构": Compressor (norm, then
//        rotary at the block start), Indexer (visibility mask, top-k),
//        Sparse Attention (window + compressed sets), 输出投影 (inverse RoPE).
//
// Readings (the same as the numpy oracle's): entry s is visible to query t iff
// (s+1)*m <= t+1; RoPE on interleaved pairs (2i, 2i+1) of the last rd dims with
// frequency theta^(-2i/rd); attention scale c^-1/2; the sink logit only in the
// denominator; window = tokens max(0, t-w+1)..t before the compressed rows;
// top-k keeps min(k, V) entries, ties to the lower index, ascending, -1 padded.
//
// Build: g++ -O3 -fopenmp -shared -fPIC (see oracle/hca_oracle_c.py).  OpenMP
// only spreads independent sequences or tokens over threads; every result is
// computed by one thread in a fixed order, so it does not depend on the thread
// count.
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

// RMSNorm over c values: x / sqrt(mean(x^2) + eps) * gamma.
void rmsnorm_row(double *x, int c, const double *gamma, double eps) {
  double ss = 0.0;
  for (int j = 0; j < c; ++j) ss += x[j] * x[j];
  const double r = 1.0 / std::sqrt(ss / c + eps);
  for (int j = 0; j < c; ++j) x[j] = x[j] * r * (gamma ? gamma[j] : 1.0);
}

// Rotate the last rd dims of x (c values) by pos (by -pos when inverse).
void rope_row(double *x, int c, long long pos, int rd, double theta, bool inverse) {
  for (int i = 0; i < rd / 2; ++i) {
    const double freq = std::pow(theta, -2.0 * i / rd);
    double ang = (double)pos * freq;
    if (inverse) ang = -ang;
    const double cs = std::cos(ang), sn = std::sin(ang);
    double &a = x[c - rd + 2 * i];
    double &b = x[c - rd + 2 * i + 1];
    const double a0 = a, b0 = b;
    a = a0 * cs - b0 * sn;
    b = a0 * sn + b0 * cs;
  }
}

}  // namespace

extern "C" {

int hco_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

// [J] Eq.(11)-(12) / (22)-(23): the n/m entries of one sequence.  Entry i,
// channel j is the softmax over the rows of block i (logit Z_a + B_a) and, for
// the overlapped CSA series (Cb != NULL) and i > 0, the rows of block i-1
// (logit Z_b + B_b), applied to the matching C values.  Inputs [n, c], biases
// [m, c], out [n/m, c].
int hco_compress(const double *Ca, const double *Za, const double *Ba, const double *Cb, const double *Zb,
                 const double *Bb, int n, int c, int m, double *out) {
  if (n < 0 || c <= 0 || m <= 0 || !Ca || !Za || !Ba || !out) return -1;
  if (Cb && (!Zb || !Bb)) return -1;
  const int E = n / m;
  std::vector<double> lg(2 * (size_t)m), vl(2 * (size_t)m);   // the logits and values of an entry's rows
  for (int i = 0; i < E; ++i) {
    for (int ch = 0; ch < c; ++ch) {
      int R = 0;
      for (int r = 0; r < m; ++r) {
        lg[R] = Za[(long long)(i * m + r) * c + ch] + Ba[(long long)r * c + ch];
        vl[R] = Ca[(long long)(i * m + r) * c + ch];
        ++R;
      }
      if (Cb && i > 0) {
        for (int r = 0; r < m; ++r) {
          lg[R] = Zb[(long long)((i - 1) * m + r) * c + ch] + Bb[(long long)r * c + ch];
          vl[R] = Cb[(long long)((i - 1) * m + r) * c + ch];
          ++R;
        }
      }
      double mx = lg[0];
      for (int r = 1; r < R; ++r) mx = std::max(mx, lg[r]);
      double den = 0.0, num = 0.0;
      for (int r = 0; r < R; ++r) {
        const double e = std::exp(lg[r] - mx);
        den += e;
        num += e * vl[r];
      }
      out[(long long)i * c + ch] = num / den;
    }
  }
  return 0;
}

// [J] §2.3.3 / [Z] Compressor: RMSNorm of each of E entries (norm != 0), then
// RoPE of its last rd dims at the entry's block start (first_entry + i) * m.
int hco_entry_epilogue(double *x, int E, int c, int m, int first_entry, const double *gamma, double eps, int rd,
                       double theta, int norm) {
  if (!x || E < 0 || c <= 0 || rd < 0 || rd > c || rd % 2) return -1;
  for (int i = 0; i < E; ++i) {
    double *row = x + (long long)i * c;
    if (norm) rmsnorm_row(row, c, gamma, eps);
    rope_row(row, c, (long long)(first_entry + i) * m, rd, theta, false);
  }
  return 0;
}

// [J] Eq.(16): I[s] = sum_h w[h] ReLU(q^I[h] . K^I[s]) for s < V.
// qI [n_hI, c_I], w [n_hI], KI [V, c_I], out [V].
int hco_index_scores(const double *qI, const double *w, const double *KI, int n_hI, int c_I, int V, double *out) {
  if (!qI || !w || (V > 0 && (!KI || !out)) || n_hI <= 0 || c_I <= 0) return -1;
  for (int s = 0; s < V; ++s) {
    double acc = 0.0;
    for (int h = 0; h < n_hI; ++h) {
      double d = 0.0;
      for (int j = 0; j < c_I; ++j) d += qI[h * c_I + j] * KI[(long long)s * c_I + j];
      acc += w[h] * (d > 0.0 ? d : 0.0);
    }
    out[s] = acc;
  }
  return 0;
}

// [J] Eq.(17): the min(k, V) highest scores, ties to the lower index; out [k]
// ascending, then -1.
int hco_topk_select(const double *scores, int V, int k, int32_t *out) {
  if (k <= 0 || !out || (V > 0 && !scores)) return -1;
  std::vector<int> ord(V);
  std::iota(ord.begin(), ord.end(), 0);
  std::sort(ord.begin(), ord.end(), [&](int a, int b) {
    if (scores[a] != scores[b]) return scores[a] > scores[b];
    return a < b;
  });
  const int n = std::min(k, V);
  std::sort(ord.begin(), ord.begin() + n);
  for (int i = 0; i < k; ++i) out[i] = i < n ? ord[i] : -1;
  return 0;
}

// [J] Eq.(18)-(19), (27), §2.3.3: shared-KV MQA for one query token.  Every
// row of rows [R, c] is both key and value for all n_h heads of q [n_h, c];
// o_h = sum_j e^{z_hj} row_j / (sum_j e^{z_hj} + e^{sink_h}), z = scale q.row,
// then the inverse RoPE of o's last rd dims at the query position t.
int hco_attend(const double *q, const double *rows, int R, const double *sink, int n_h, int c, double scale,
               long long t, int rd, double theta, double *out) {
  if (!q || !sink || !out || (R > 0 && !rows) || n_h <= 0 || c <= 0) return -1;
  std::vector<double> z(R > 0 ? R : 1);
  for (int h = 0; h < n_h; ++h) {
    double M = sink[h];
    for (int r = 0; r < R; ++r) {
      double d = 0.0;
      for (int j = 0; j < c; ++j) d += q[(long long)h * c + j] * rows[(long long)r * c + j];
      z[r] = d * scale;
      M = std::max(M, z[r]);
    }
    double den = std::exp(sink[h] - M);
    double *o = out + (long long)h * c;
    for (int j = 0; j < c; ++j) o[j] = 0.0;
    for (int r = 0; r < R; ++r) {
      const double e = std::exp(z[r] - M);
      den += e;
      for (int j = 0; j < c; ++j) o[j] += e * rows[(long long)r * c + j];
    }
    for (int j = 0; j < c; ++j) o[j] /= den;
    rope_row(o, c, t, rd, theta, true);
  }
  return 0;
}

// Rows of a cache as the GPU stores them, decoded exactly to double: dtype 0
// float64, 1 bfloat16 bits, 2 fp8 e4m3 codes times a per-row fp32 scale.
struct hco_rows {
  const void *p;
  int dtype;
  const float *scale;   // [rows] for dtype 2
  long long n_rows;     // rows per sequence (the stride between sequences)
};

}  // extern "C"

namespace {

// bfloat16: the upper 16 bits of an IEEE binary32.
double bf16_to_double(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// e4m3 (OCP FP8): sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0
// is subnormal (m/8 * 2^-6); 0x7F / 0xFF are NaN; no infinities.
double e4m3_to_double(uint8_t v) {
  const int sgn = v >> 7, e = (v >> 3) & 15, m = v & 7;
  if (e == 15 && m == 7) return std::nan("");
  const double mag = e == 0 ? std::ldexp((double)m / 8.0, -6) : std::ldexp(1.0 + (double)m / 8.0, e - 7);
  return sgn ? -mag : mag;
}

void get_row(const hco_rows &r, long long seq, long long i, int c, double *out) {
  const long long row = seq * r.n_rows + i;
  if (r.dtype == 0) {
    std::memcpy(out, static_cast<const double *>(r.p) + row * c, sizeof(double) * c);
  } else if (r.dtype == 1) {
    const uint16_t *b = static_cast<const uint16_t *>(r.p) + row * c;
    for (int j = 0; j < c; ++j) out[j] = bf16_to_double(b[j]);
  } else {
    const uint8_t *b = static_cast<const uint8_t *>(r.p) + row * c;
    const double s = (double)r.scale[row];
    for (int j = 0; j < c; ++j) out[j] = e4m3_to_double(b[j]) * s;
  }
}

}  // namespace

extern "C" {

// One query token of sequence `seq` of a CSA (kind 1) or HCA (kind 0)
// attention, from the caches: the window rows win_idx[0..nw) of `win` (in
// position order: tokens max(0, t-w+1)..t), the visible compressed entries of
// `comp` (V = (t+1)/m); CSA also scores and selects (q^I [n_hI, c_I], w
// [n_hI] in double, keys `KI`) and writes the selection to idx_out [k] (may be
// NULL).  q [n_h, c]; out [n_h, c].
int hco_token(int kind, long long seq, const double *q, hco_rows win, const int32_t *win_idx, int nw, hco_rows comp,
              int m, int k, const double *qI, const double *w, hco_rows KI, int n_hI, int c_I, const double *sink,
              int n_h, int c, int rd, double theta, long long t, double *out, int32_t *idx_out) {
  const int V = (int)((t + 1) / m);
  std::vector<int> sel;
  if (kind == 1) {
    std::vector<double> keys((size_t)(V > 0 ? V : 1) * c_I), sc(V > 0 ? V : 1);
    for (int s = 0; s < V; ++s) get_row(KI, seq, s, c_I, keys.data() + (size_t)s * c_I);
    std::vector<int32_t> idx(k);
    if (hco_index_scores(qI, w, keys.data(), n_hI, c_I, V, sc.data()) || hco_topk_select(sc.data(), V, k, idx.data()))
      return -1;
    for (int i = 0; i < k; ++i)
      if (idx[i] >= 0) sel.push_back(idx[i]);
    if (idx_out) std::memcpy(idx_out, idx.data(), sizeof(int32_t) * k);
  } else {
    for (int s = 0; s < V; ++s) sel.push_back(s);
  }
  const int R = nw + (int)sel.size();
  std::vector<double> rows((size_t)(R > 0 ? R : 1) * c);
  for (int i = 0; i < nw; ++i) get_row(win, seq, win_idx[i], c, rows.data() + (size_t)i * c);
  for (size_t i = 0; i < sel.size(); ++i) get_row(comp, seq, sel[i], c, rows.data() + (size_t)(nw + i) * c);
  return hco_attend(q, rows.data(), R, sink, n_h, c, 1.0 / std::sqrt((double)c), t, rd, theta, out);
}

// A decode step of B sequences at position t, the sequences spread over the
// OpenMP threads: sequence b's query q + b n_h c, window rows win_idx (ring
// slots in position order, shared by all sequences), caches at sequence b,
// q^I + b n_hI c_I, w + b n_hI; out + b n_h c.  Returns 0, or -1 if any
// sequence failed.
int hco_decode_batch(int kind, int B, const double *q, hco_rows win, const int32_t *win_idx, int nw, hco_rows comp,
                     int m, int k, const double *qI, const double *w, hco_rows KI, int n_hI, int c_I,
                     const double *sink, int n_h, int c, int rd, double theta, long long t, double *out) {
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int b = 0; b < B; ++b) {
    bad |= hco_token(kind, b, q + (size_t)b * n_h * c, win, win_idx, nw, comp, m, k,
                     kind == 1 ? qI + (size_t)b * n_hI * c_I : nullptr, kind == 1 ? w + (size_t)b * n_hI : nullptr, KI,
                     n_hI, c_I, sink, n_h, c, rd, theta, t, out + (size_t)b * n_h * c, nullptr) != 0;
  }
  return bad ? -1 : 0;
}

// Prefill attention of a list of query tokens of sequence `seq` (OpenMP over
// the tokens): token ts[i] attends its window rows (token rows of `win`) and
// its compressed set; q [n_tok, n_h, c] holds the listed tokens' queries in
// list order, q^I / w likewise (CSA).
int hco_prefill_tokens(int kind, long long seq, int n_tok, const long long *ts, const double *q, hco_rows win,
                       int w_len, hco_rows comp, int m, int k, const double *qI, const double *w, hco_rows KI,
                       int n_hI, int c_I, const double *sink, int n_h, int c, int rd, double theta, double *out) {
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int i = 0; i < n_tok; ++i) {
    const long long t = ts[i];
    const long long t0 = t - w_len + 1 > 0 ? t - w_len + 1 : 0;
    const int nw = w_len > 0 ? (int)(t - t0 + 1) : 0;
    std::vector<int32_t> wi(nw > 0 ? nw : 1);
    for (int j = 0; j < nw; ++j) wi[j] = (int32_t)(t0 + j);
    bad |= hco_token(kind, seq, q + (size_t)i * n_h * c, win, wi.data(), nw, comp, m, k,
                     kind == 1 ? qI + (size_t)i * n_hI * c_I : nullptr, kind == 1 ? w + (size_t)i * n_hI : nullptr, KI,
                     n_hI, c_I, sink, n_h, c, rd, theta, t, out + (size_t)i * n_h * c, nullptr) != 0;
  }
  return bad ? -1 : 0;
}

}  // extern "C"
