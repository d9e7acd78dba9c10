// compress.cu -- block compression of KV entries.
//
// CSA (juejin "DeepSeek-V4 技术报告简要解读" §2.3.1(a), Eq.(11)-(12)): entry i,
// channel ch is the softmax over the 2m logits {Z_a rows of block i + B_a} U
// {Z_b rows of block i-1 + B_b} applied to the matching C_a / C_b values.
// HCA (§2.3.2, Eq.(22)-(23)): softmax over the m' rows of block i (+ B).
// Epilogue (§2.3.3; 1zeryu "DeepSeek-V4：算法架构", Compressor): RMSNorm of the
// entry, RoPE of its last rd dims at the block start i*m, and for fp8 output a
// per-entry amax/448 scale.
//
// HBM-bound: every C/Z element is read once (16-byte vector loads), each entry
// written once.  A thread owns 8 channels and a slice of the block's rows and
// keeps an online (running max) softmax per channel; slices are merged in
// shared memory.  The decode branch keeps the block's rows in a caller-owned
// fp32 state and emits an entry when a block completes.
#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {

constexpr int kThreads = 256;

template <typename Tin>
__device__ __forceinline__ const Tin *row_ptr(const void *base, long long seq_stride,
                                             long long row_stride, int b, long long tok) {
  return reinterpret_cast<const Tin *>(base) + (long long)b * seq_stride + tok * row_stride;
}

// Write one finished entry (8 channels per thread) with the epilogue applied.
// `vals` are this thread's 8 channel values; `red` is shared scratch of at
// least `cv` floats per entry slot.  All threads of the block must call it.
template <typename Tout>
struct EntryWriter;

template <>
struct EntryWriter<float> {
  static __device__ void put(float *row, int ch0, const float (&v)[8], float) { store8(row + ch0, v); }
};
template <>
struct EntryWriter<__nv_bfloat16> {
  static __device__ void put(__nv_bfloat16 *row, int ch0, const float (&v)[8], float) {
    store8(row + ch0, v);
  }
};
template <>
struct EntryWriter<uint8_t> {
  static __device__ void put(uint8_t *row, int ch0, const float (&v)[8], float inv_scale) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      lo |= (uint32_t)__nv_cvt_float_to_fp8(v[j] * inv_scale, __NV_SATFINITE, __NV_E4M3) << (8 * j);
      hi |= (uint32_t)__nv_cvt_float_to_fp8(v[4 + j] * inv_scale, __NV_SATFINITE, __NV_E4M3)
            << (8 * j);
    }
    *reinterpret_cast<uint2 *>(row + ch0) = make_uint2(lo, hi);
  }
};

// Per-entry epilogue for `epb` entries handled by one block: norm, rope,
// fp8 scale, store.  Thread t with active=true owns channels [ch0, ch0+8) of
// entry slot `slot`.
template <typename Tout>
__device__ void entry_epilogue(const CompressParams &p, float (&v)[8], bool active, int slot,
                               int cvi, int cv, int b, long long entry, long long pos,
                               float *red /* [epb * cv] */, float *red2) {
  const int ch0 = cvi * 8;
  if (p.flags & HCA_COMPRESS_NORM) {
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss += v[j] * v[j];
    if (active) red[slot * cv + cvi] = ss;
    __syncthreads();
    if (active) {
      float tot = 0.f;
      for (int j = 0; j < cv; ++j) tot += red[slot * cv + j];
      const float r = rsqrtf(tot / (float)p.width + p.eps);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] *= r * (p.gamma ? p.gamma[ch0 + j] : 1.f);
    }
    __syncthreads();
  }
  if ((p.flags & HCA_COMPRESS_ROPE) && p.rd > 0 && active && ch0 >= p.width - p.rd) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float s, c;
      rope_sincos_tab(p.rope_freq, pos, (ch0 - (p.width - p.rd)) / 2 + j, p.rd, p.theta, &s, &c);
      const float a = v[2 * j], bb = v[2 * j + 1];
      v[2 * j] = a * c - bb * s;
      v[2 * j + 1] = a * s + bb * c;
    }
  }
  float inv_scale = 1.f;
  if (p.out_dtype == HCA_FP8E4M3) {
    float am = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(v[j]));
    if (active) red2[slot * cv + cvi] = am;
    __syncthreads();
    if (active) {
      float tot = 0.f;
      for (int j = 0; j < cv; ++j) tot = fmaxf(tot, red2[slot * cv + j]);
      tot = fmaxf(tot, 1e-12f);
      const float scale = tot / 448.f;
      inv_scale = 1.f / scale;
      if (cvi == 0) p.out_scale[(long long)b * p.out_seq_stride + entry] = scale;
    }
    __syncthreads();
  }
  if (active) {
    Tout *row = reinterpret_cast<Tout *>(p.out) + ((long long)b * p.out_seq_stride + entry) * p.width;
    EntryWriter<Tout>::put(row, ch0, v, inv_scale);
  }
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads)
compress_prefill_kernel(CompressParams p, int epb, int rg) {
  extern __shared__ float sm[];
  const int cv = p.width / 8;
  const int tpe = kThreads / epb;
  const int tid = threadIdx.x;
  const int slot = tid / tpe;
  const int local = tid % tpe;
  const int cvi = local % cv;
  const int rgi = local / cv;
  const int b = blockIdx.y;
  const int E = p.n / p.m;
  const long long entry = p.e_first + (long long)blockIdx.x * epb + slot;
  const bool valid = entry < E && rgi < rg;
  const int R = (p.overlap && entry > 0) ? 2 * p.m : p.m;

  float mx[8], sum[8], acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) { mx[j] = -INFINITY; sum[j] = 0.f; acc[j] = 0.f; }

  if (valid) {
    for (int r = rgi; r < R; r += rg) {
      const bool a_series = r < p.m;
      const int j = a_series ? r : r - p.m;
      const long long tok = a_series ? entry * p.m + j : (entry - 1) * p.m + j;
      const Tin *zp = row_ptr<Tin>(a_series ? p.Za : p.Zb, p.seq_stride, p.row_stride, b, tok);
      const Tin *cp = row_ptr<Tin>(a_series ? p.Ca : p.Cb, p.seq_stride, p.row_stride, b, tok);
      const float *bp = (a_series ? p.Ba : p.Bb) + (long long)j * p.width + cvi * 8;
      float z[8], cval[8];
      load8(zp + cvi * 8, z);
      load8(cp + cvi * 8, cval);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float l = z[q] + bp[q];
        const float nm = fmaxf(mx[q], l);
        const float sc = __expf(mx[q] - nm);   // mx = -inf on the first row -> 0
        const float e = __expf(l - nm);
        sum[q] = sum[q] * sc + e;
        acc[q] = acc[q] * sc + e * cval[q];
        mx[q] = nm;
      }
    }
  }
  // merge the row-group partials of each entry slot
  float *pm = sm;                       // [kThreads][8]
  float *ps = sm + kThreads * 8;        // [kThreads][8]
  float *pa = sm + 2 * kThreads * 8;    // [kThreads][8]
  float *red = sm + 3 * kThreads * 8;   // [epb * cv]
  float *red2 = red + epb * cv;         // [epb * cv]
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    pm[tid * 8 + q] = mx[q];
    ps[tid * 8 + q] = sum[q];
    pa[tid * 8 + q] = acc[q];
  }
  __syncthreads();
  float v[8];
  const bool active = valid && rgi == 0;
  if (active) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float M = -INFINITY;
      for (int g = 0; g < rg; ++g) M = fmaxf(M, pm[(slot * tpe + g * cv + cvi) * 8 + q]);
      float S = 0.f, A = 0.f;
      for (int g = 0; g < rg; ++g) {
        const int t = (slot * tpe + g * cv + cvi) * 8 + q;
        const float sc = (pm[t] == -INFINITY) ? 0.f : __expf(pm[t] - M);
        S += ps[t] * sc;
        A += pa[t] * sc;
      }
      v[q] = A / S;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = 0.f;
  }
  entry_epilogue<Tout>(p, v, active, slot, cvi, cv, b, entry - p.e_first, (p.e_pos0 + entry) * p.m, red, red2);
}

// Prefill with many entries, for widths whose 8-channel groups tile a warp
// (c/8 a power of two up to 32, or a multiple of 32 up to 256): a thread owns 8 channels of one
// entry and all of the entry's rows (no partial softmaxes to merge), loading
// kRowBatch rows at a time with all of their loads in flight; the entry's
// sums of squares and maxima are reduced by shuffles within its lanes and,
// when the entry spans several warps, through shared memory under a named
// barrier of just those warps -- no block-wide barrier.
constexpr int kRowBatch = 4;

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) compress_prefill_rows_kernel(CompressParams p) {
  __shared__ float xbuf[2][kThreads / 32];
  const int cv = p.width / 8;
  const int epc = kThreads / cv;                 // entries per block
  const int tid = threadIdx.x;
  const int slot = tid / cv, cvi = tid - slot * cv;
  const int b = blockIdx.y;
  const int E = p.n / p.m;
  const long long entry = p.e_first + (long long)blockIdx.x * epc + slot;
  const bool valid = entry < E;
  const int R = (p.overlap && entry > 0) ? 2 * p.m : p.m;
  float mx[8], sum[8], acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) { mx[j] = -INFINITY; sum[j] = 0.f; acc[j] = 0.f; }
  if (valid) {
    for (int r0 = 0; r0 < R; r0 += kRowBatch) {
      float z[kRowBatch][8], cval[kRowBatch][8];
#pragma unroll
      for (int k = 0; k < kRowBatch; ++k) {
        const int r = r0 + k;
        if (r < R) {
          const bool a_series = r < p.m;
          const int j = a_series ? r : r - p.m;
          const long long tok = a_series ? entry * p.m + j : (entry - 1) * p.m + j;
          load8(row_ptr<Tin>(a_series ? p.Za : p.Zb, p.seq_stride, p.row_stride, b, tok) + cvi * 8, z[k]);
          load8(row_ptr<Tin>(a_series ? p.Ca : p.Cb, p.seq_stride, p.row_stride, b, tok) + cvi * 8, cval[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < kRowBatch; ++k) {
        const int r = r0 + k;
        if (r < R) {
          const bool a_series = r < p.m;
          const int j = a_series ? r : r - p.m;
          const float *bp = (a_series ? p.Ba : p.Bb) + (long long)j * p.width + cvi * 8;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float l = z[k][q] + bp[q];
            const float nm = fmaxf(mx[q], l);
            const float sc = __expf(mx[q] - nm);   // mx = -inf on the first row -> 0
            const float e = __expf(l - nm);
            sum[q] = sum[q] * sc + e;
            acc[q] = acc[q] * sc + e * cval[k][q];
            mx[q] = nm;
          }
        }
      }
    }
  }
  float v[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) v[q] = valid ? acc[q] / sum[q] : 0.f;
  // reduction over the entry's cv lanes (use 0: sums, 1: maxima)
  auto reduce = [&](float x, bool is_max, int use) -> float {
    const int g = cv < 32 ? cv : 32;
    for (int o = g / 2; o > 0; o >>= 1) {
      const float y = __shfl_xor_sync(0xffffffffu, x, o);
      x = is_max ? fmaxf(x, y) : x + y;
    }
    if (cv <= 32) return x;
    const int wpe = cv / 32, w = tid >> 5;       // warps per entry, this warp
    if ((tid & 31) == 0) xbuf[use][w] = x;
    asm volatile("bar.sync %0, %1;" ::"r"(1 + slot), "r"(cv) : "memory");
    float t = is_max ? 0.f : 0.f;
    for (int i = 0; i < wpe; ++i) {
      const float y = xbuf[use][slot * wpe + i];
      t = is_max ? fmaxf(t, y) : t + y;
    }
    return t;
  };
  const int ch0 = cvi * 8;
  if (p.flags & HCA_COMPRESS_NORM) {
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss += v[j] * v[j];
    const float tot = reduce(ss, false, 0);
    const float rn = rsqrtf(tot / (float)p.width + p.eps);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] *= rn * (p.gamma ? p.gamma[ch0 + j] : 1.f);
  }
  if ((p.flags & HCA_COMPRESS_ROPE) && p.rd > 0 && ch0 >= p.width - p.rd) {
    const long long pos = (p.e_pos0 + entry) * p.m;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float sn, cs;
      rope_sincos_tab(p.rope_freq, pos, (ch0 - (p.width - p.rd)) / 2 + j, p.rd, p.theta, &sn, &cs);
      const float a = v[2 * j], bb = v[2 * j + 1];
      v[2 * j] = a * cs - bb * sn;
      v[2 * j + 1] = a * sn + bb * cs;
    }
  }
  float inv_scale = 1.f;
  if (p.out_dtype == HCA_FP8E4M3) {
    float am = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(v[j]));
    const float tot = fmaxf(reduce(am, true, 1), 1e-12f);
    const float scale = tot / 448.f;
    inv_scale = 1.f / scale;
    if (valid && cvi == 0) p.out_scale[(long long)b * p.out_seq_stride + (entry - p.e_first)] = scale;
  }
  if (valid) {
    Tout *row = reinterpret_cast<Tout *>(p.out) + ((long long)b * p.out_seq_stride + (entry - p.e_first)) * p.width;
    EntryWriter<Tout>::put(row, ch0, v, inv_scale);
  }
}

// Prefill leaves the state ready for decode at position n (rows of the last
// complete block and of the incomplete tail; empty rows (0, -inf)).
template <typename Tin>
__global__ void compress_state_prefill_kernel(CompressParams p) {
  const int b = blockIdx.y;
  const int m = p.m, W = p.width;
  const int cutoff = (p.n / m) * m, rem = p.n - cutoff;
  const int R = p.overlap ? 2 * m : m;
  const int C = p.overlap ? 2 * W : W;
  const long long total = (long long)R * C;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / C), col = (int)(e % C);
    long long tok = -1;
    int j = 0;
    if (p.overlap) {
      if (r < m) { if (cutoff >= m) { tok = cutoff - m + r; j = r; } }
      else if (r - m < rem) { tok = cutoff + (r - m); j = r - m; }
    } else if (r < rem) { tok = cutoff + r; j = r; }
    float kv = 0.f, sc = -INFINITY;
    if (tok >= 0) {
      const bool b_half = p.overlap && col < W;
      const int ch = p.overlap ? (b_half ? col : col - W) : col;
      const Tin *cp = row_ptr<Tin>(b_half ? p.Cb : p.Ca, p.seq_stride, p.row_stride, b, tok);
      const Tin *zp = row_ptr<Tin>(b_half ? p.Zb : p.Za, p.seq_stride, p.row_stride, b, tok);
      const float *bp = b_half ? p.Bb : p.Ba;
      kv = Elt<Tin>::load(cp + ch);
      sc = Elt<Tin>::load(zp + ch) + bp[(long long)j * W + ch];
    }
    const long long off = ((long long)b * R + r) * C + col;
    p.state_kv[off] = kv;
    p.state_score[off] = sc;
  }
}

// Decode: one block per sequence.  `sm` holds (width + width/4) floats.
template <typename Tin, typename Tout>
__device__ __forceinline__ void compress_decode_block(const CompressParams &p, int pos, int b, float *sm) {
  const int m = p.m, W = p.width;
  const int R = p.overlap ? 2 * m : m;
  const int C = p.overlap ? 2 * W : W;
  const int j = pos % m;
  float *skv = p.state_kv + (long long)b * R * C;
  float *ssc = p.state_score + (long long)b * R * C;
  const Tin *ca = row_ptr<Tin>(p.Ca, p.seq_stride, 0, b, 0);
  const Tin *za = row_ptr<Tin>(p.Za, p.seq_stride, 0, b, 0);
  // 1. store the token's rows (value, logit + bias)
  for (int ch = threadIdx.x; ch < W; ch += kThreads) {
    if (p.overlap) {
      const Tin *cb = row_ptr<Tin>(p.Cb, p.seq_stride, 0, b, 0);
      const Tin *zb = row_ptr<Tin>(p.Zb, p.seq_stride, 0, b, 0);
      const long long row = (long long)(m + j) * C;
      skv[row + ch] = Elt<Tin>::load(cb + ch);
      ssc[row + ch] = Elt<Tin>::load(zb + ch) + p.Bb[(long long)j * W + ch];
      skv[row + W + ch] = Elt<Tin>::load(ca + ch);
      ssc[row + W + ch] = Elt<Tin>::load(za + ch) + p.Ba[(long long)j * W + ch];
    } else {
      const long long row = (long long)j * C;
      skv[row + ch] = Elt<Tin>::load(ca + ch);
      ssc[row + ch] = Elt<Tin>::load(za + ch) + p.Ba[(long long)j * W + ch];
    }
  }
  if ((pos + 1) % m != 0) return;   // uniform across the block
  __syncthreads();
  // 2. emit the entry: per channel softmax over the block's rows
  float *ent = sm;                   // [W]
  float *red = sm + W;               // [W / 8]
  float *red2 = red + W / 8;         // [W / 8]
  // one online pass over the block's rows, 8 rows per step with their loads
  // issued together (an HCA block has 128 rows)
  for (int ch = threadIdx.x; ch < W; ch += kThreads) {
    float M = -INFINITY, S = 0.f, A = 0.f;
    for (int r0 = 0; r0 < m; r0 += 8) {
      float za[8], va[8], zb[8], vb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int r = r0 + u;
        za[u] = -INFINITY; va[u] = 0.f; zb[u] = -INFINITY; vb[u] = 0.f;
        if (r < m) {
          if (p.overlap) {
            zb[u] = ssc[(long long)r * C + ch];
            vb[u] = skv[(long long)r * C + ch];
            za[u] = ssc[(long long)(m + r) * C + W + ch];
            va[u] = skv[(long long)(m + r) * C + W + ch];
          } else {
            za[u] = ssc[(long long)r * C + ch];
            va[u] = skv[(long long)r * C + ch];
          }
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int u = 0; u < 8; ++u) mx = fmaxf(mx, fmaxf(za[u], zb[u]));
      if (mx == -INFINITY) continue;
      const float Mn = fmaxf(M, mx);
      const float sc = __expf(M - Mn);   // 0 while M is still -inf
      S *= sc;
      A *= sc;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float ea = __expf(za[u] - Mn), eb = __expf(zb[u] - Mn);
        S += ea + eb;
        A += ea * va[u] + eb * vb[u];
      }
      M = Mn;
    }
    ent[ch] = A / S;
  }
  __syncthreads();
  const int cv = W / 8;
  const bool active = threadIdx.x < cv;
  float v[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) v[q] = active ? ent[threadIdx.x * 8 + q] : 0.f;
  const long long entry = pos / m;
  // the entry goes to out slot entry - e_first (e_first = entry: a one-row scratch)
  entry_epilogue<Tout>(p, v, active, 0, active ? threadIdx.x : 0, cv, b, entry - p.e_first,
                       (long long)(pos + 1 - m), red, red2);
  __syncthreads();
  // 3. shift the state: the finished block becomes the previous block
  for (long long e = threadIdx.x; e < (long long)m * C; e += kThreads) {
    if (p.overlap) {
      skv[e] = skv[(long long)m * C + e];
      ssc[e] = ssc[(long long)m * C + e];
      skv[(long long)m * C + e] = 0.f;
      ssc[(long long)m * C + e] = -INFINITY;
    } else {
      skv[e] = 0.f;
      ssc[e] = -INFINITY;
    }
  }
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) compress_decode_kernel(CompressParams p, int pos) {
  extern __shared__ float sm[];
  compress_decode_block<Tin, Tout>(p, pos, blockIdx.x, sm);
}

// One decode token of one layer in one launch: blockIdx.y = 0 advances the
// main compressor, 1 the indexer compressor (when present), the last part
// writes the token's window row into the ring.  blockIdx.x = sequence.
template <typename Tin, typename TA, typename TB, typename Tw>
__global__ void __launch_bounds__(kThreads) decode_ingest_kernel(CompressParams pa, CompressParams pb, int has_b,
                                                                 IngestRing ring, int pos) {
  extern __shared__ float sm[];
  const int b = blockIdx.x, part = blockIdx.y;
  const unsigned long long st_entry = global_ns();
  pdl_trigger();   // the layer's next kernel may start its prologue
  if (part == 0 && pa.B > 0) {
    compress_decode_block<Tin, TA>(pa, pos, b, sm);
  } else if (part == 1 && has_b) {
    compress_decode_block<Tin, TB>(pb, pos, b, sm);
  } else if (ring.ring) {
    const Tw *row = reinterpret_cast<const Tw *>(ring.row) + (long long)b * ring.c;
    Tw *dst = reinterpret_cast<Tw *>(ring.ring) + ((long long)b * ring.w + ring.slot) * ring.c;
    for (int col = threadIdx.x; col < ring.c; col += kThreads) dst[col] = row[col];
  }
  if (step_trace_on()) {
    __syncthreads();
    if (threadIdx.x == 0) step_trace_record(ST_INGEST, st_entry, st_entry);
  }
}

template <typename Tin>
int launch_prefill_t(const CompressParams &p, cudaStream_t s) {
  const int cv = p.width / 8;
  const long long E_w = p.n / p.m - p.e_first;   // entries written
  // a thread per (entry, 8 channels) when that gives half the SMs a block;
  // few long entries (HCA) split their rows over row groups instead
  if ((((cv & (cv - 1)) == 0 && cv <= 32) || (cv % 32 == 0 && cv <= kThreads)) &&
      (long long)p.B * ((E_w + kThreads / cv - 1) / (kThreads / cv)) >= num_sms() / 2) {
    const long long E = E_w;
    const int epc = kThreads / cv;
    dim3 grid((unsigned)((E + epc - 1) / epc), p.B);
    LaunchScope ls_("compress_prefill", s);
    switch (p.out_dtype) {
      case HCA_F32: compress_prefill_rows_kernel<Tin, float><<<grid, kThreads, 0, s>>>(p); break;
      case HCA_BF16: compress_prefill_rows_kernel<Tin, __nv_bfloat16><<<grid, kThreads, 0, s>>>(p); break;
      default: compress_prefill_rows_kernel<Tin, uint8_t><<<grid, kThreads, 0, s>>>(p); break;
    }
    return ls_.done();
  }
  const int R = p.overlap ? 2 * p.m : p.m;
  // entries per block: give each entry about cv * R threads, at most kThreads
  int epb = 1;
  while (epb < 32 && cv * R * epb * 2 <= kThreads && cv * epb * 2 <= kThreads) epb *= 2;
  const int tpe = kThreads / epb;
  int rg = tpe / cv;
  if (rg > R) rg = R;
  const long long E = p.n / p.m - p.e_first;   // entries written
  if (E <= 0) return HCA_OK;
  dim3 grid((unsigned)((E + epb - 1) / epb), p.B);
  const size_t smem = (size_t)(3 * kThreads * 8 + 2 * epb * cv) * sizeof(float);
  LaunchScope ls_("compress_prefill", s);
  switch (p.out_dtype) {
    case HCA_F32: compress_prefill_kernel<Tin, float><<<grid, kThreads, smem, s>>>(p, epb, rg); break;
    case HCA_BF16: compress_prefill_kernel<Tin, __nv_bfloat16><<<grid, kThreads, smem, s>>>(p, epb, rg); break;
    default: compress_prefill_kernel<Tin, uint8_t><<<grid, kThreads, smem, s>>>(p, epb, rg); break;
  }
  return ls_.done();
}

template <typename Tin>
int launch_decode_t(const CompressParams &p, int pos, cudaStream_t s) {
  const size_t smem = (size_t)(p.width + 2 * (p.width / 8)) * sizeof(float);
  LaunchScope ls_("compress_decode", s);
  switch (p.out_dtype) {
    case HCA_F32: compress_decode_kernel<Tin, float><<<p.B, kThreads, smem, s>>>(p, pos); break;
    case HCA_BF16: compress_decode_kernel<Tin, __nv_bfloat16><<<p.B, kThreads, smem, s>>>(p, pos); break;
    default: compress_decode_kernel<Tin, uint8_t><<<p.B, kThreads, smem, s>>>(p, pos); break;
  }
  return ls_.done();
}

}  // namespace

// FP4 keys (HCA_FP4): the entries are written in bf16 and then rotated and
// FP4-quantised in place (Hadamard, blocks of 32; width 64).
int launch_decode_ingest_t(const CompressParams *pa, const CompressParams *pb, CompressParams a, CompressParams bb,
                           const IngestRing &ring, int B, int pos, cudaStream_t s);

int launch_compress_prefill(const CompressParams &p0, cudaStream_t s) {
  CompressParams p = p0;
  if (p.out_dtype == HCA_FP4) p.out_dtype = HCA_BF16;
  const int rc = p.in_dtype == HCA_F32 ? launch_prefill_t<float>(p, s) : launch_prefill_t<__nv_bfloat16>(p, s);
  if (rc || p0.out_dtype != HCA_FP4) return rc;
  const long long E = p.n / p.m - p.e_first;
  if (E <= 0) return HCA_OK;
  return launch_fp4_rotate_quant(p.out, HCA_BF16, (long long)p.B * E, p.out, s, E, p.out_seq_stride);
}

int launch_compress_state_prefill(const CompressParams &p, cudaStream_t s) {
  dim3 grid(16, p.B);
  LaunchScope ls_("compress_state", s);
  if (p.in_dtype == HCA_F32)
    compress_state_prefill_kernel<float><<<grid, 256, 0, s>>>(p);
  else
    compress_state_prefill_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  return ls_.done();
}

int launch_compress_decode(const CompressParams &p0, int pos, cudaStream_t s) {
  CompressParams p = p0;
  if (p.out_dtype == HCA_FP4) p.out_dtype = HCA_BF16;
  const int rc = p.in_dtype == HCA_F32 ? launch_decode_t<float>(p, pos, s) : launch_decode_t<__nv_bfloat16>(p, pos, s);
  if (rc || p0.out_dtype != HCA_FP4 || (pos + 1) % p.m != 0) return rc;
  // the entry this token completed, one row per sequence
  void *row = static_cast<__nv_bfloat16 *>(p.out) + (long long)(pos / p.m) * p.width;
  return launch_fp4_rotate_quant(row, HCA_BF16, p.B, row, s, 1, p.out_seq_stride);
}

int launch_decode_ingest(const CompressParams *pa, const CompressParams *pb, const IngestRing &ring, int B, int pos,
                         cudaStream_t s) {
  const int parts = (pa ? 1 : 0) + (pb ? 1 : 0) + (ring.ring ? 1 : 0);
  if (parts == 0 || B == 0) return HCA_OK;
  CompressParams a = pa ? *pa : CompressParams{};
  CompressParams bb = pb ? *pb : CompressParams{};
  // FP4 indexer keys: the emitted key is written in bf16, then rotated and
  // FP4-quantised in place by a second launch (emitting steps only)
  const bool fp4 = pb && bb.out_dtype == HCA_FP4;
  if (fp4) bb.out_dtype = HCA_BF16;
  const int rc = launch_decode_ingest_t(pa ? &a : nullptr, pb ? &bb : nullptr, a, bb, ring, B, pos, s);
  if (rc || !fp4 || (pos + 1) % bb.m != 0) return rc;
  void *row = static_cast<__nv_bfloat16 *>(bb.out) + (long long)(pos / bb.m) * bb.width;
  return launch_fp4_rotate_quant(row, HCA_BF16, B, row, s, 1, bb.out_seq_stride);
}

int launch_decode_ingest_t(const CompressParams *pa, const CompressParams *pb, CompressParams a, CompressParams bb,
                           const IngestRing &ring, int B, int pos, cudaStream_t s) {
  if (!pa) a.B = 0;
  // part indices: 0 = main (may be empty), 1 = indexer (may be absent), last = ring
  const int ny = pb ? (ring.ring ? 3 : 2) : (ring.ring ? 2 : 1);
  const int wmax = (pa ? a.width : 0) > (pb ? bb.width : 0) ? (pa ? a.width : 0) : (pb ? bb.width : 0);
  const size_t smem = (size_t)(wmax + 2 * (wmax / 8)) * sizeof(float);
  const hca_dtype ta = pa ? a.out_dtype : (ring.dtype == HCA_F32 ? HCA_F32 : HCA_BF16);
  const hca_dtype tb = pb ? bb.out_dtype : ta;
  const bool in32 = (pa ? a.in_dtype : (pb ? bb.in_dtype : HCA_F32)) == HCA_F32;
  if (!in32) return fail(HCA_ERR_UNSUPPORTED, "decode ingest takes fp32 compressor inputs");
  if (ring.ring && ring.dtype != ta) return fail(HCA_ERR_UNSUPPORTED, "window dtype must match the entry dtype");
  const dim3 grid(B, ny);
  LaunchScope ls_("decode_ingest", s);
  const int hb = pb ? 1 : 0;
  if (ta == HCA_F32 && tb == HCA_F32)
    decode_ingest_kernel<float, float, float, float><<<grid, kThreads, smem, s>>>(a, bb, hb, ring, pos);
  else if (ta == HCA_BF16 && tb == HCA_BF16)
    decode_ingest_kernel<float, __nv_bfloat16, __nv_bfloat16, __nv_bfloat16><<<grid, kThreads, smem, s>>>(a, bb, hb, ring, pos);
  else if (ta == HCA_BF16 && tb == HCA_FP8E4M3)
    decode_ingest_kernel<float, __nv_bfloat16, uint8_t, __nv_bfloat16><<<grid, kThreads, smem, s>>>(a, bb, hb, ring, pos);
  else if (ta == HCA_F32 && tb == HCA_FP8E4M3)
    decode_ingest_kernel<float, float, uint8_t, float><<<grid, kThreads, smem, s>>>(a, bb, hb, ring, pos);
  else if (ta == HCA_F32 && tb == HCA_BF16)
    decode_ingest_kernel<float, float, __nv_bfloat16, float><<<grid, kThreads, smem, s>>>(a, bb, hb, ring, pos);
  else
    decode_ingest_kernel<float, __nv_bfloat16, float, __nv_bfloat16><<<grid, kThreads, smem, s>>>(a, bb, hb, ring, pos);
  return ls_.done();
}

int step_trace_set_compress(void *buf, unsigned long long cap) { return step_trace_set_here(buf, cap); }

}  // namespace hca
