// index_topk.cu -- lightning-indexer scores and per-query top-k selection.
//
// Score (juejin "DeepSeek-V4 技术报告简要解读" §2.3.1(b), Eq.(16); 1zeryu
// "DeepSeek-V4：算法架构", Indexer):  I[t,s] = sum_h w[t,h] ReLU(q^I[t,h].K^I[s])
// for the entries visible to t ((s+1)*m <= t+1).
// Selection (Eq.(17)): the min(k, V_t) highest scores, ties broken towards the
// lower entry index, emitted in ascending index order and padded with -1.
//
// The selection is exact on the order-preserving uint32 image of the fp32
// scores, by one of four kernels chosen by shape: many rows (prefill) take a
// warp per row (sampled thresholds, one pass, radix select within the band);
// a few rows of up to 32768 keys a CTA per row (the row in registers); a few
// longer rows a thread-block cluster per row; the general fallback is a
// segmented radix select (digits of 11, 11 and 10 bits) by thread-block
// clusters that sum their histograms through distributed shared memory.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {

// ------------------------------------------------------------------ scores
// SIMT scorer: one thread per entry, a block covers 128 entries x QB queries.
// Keys are read once per block and reused for its QB queries.
constexpr int kScoreThreads = 128;
constexpr int kQB = 8;

template <typename Tq, typename Tk>
__global__ void __launch_bounds__(kScoreThreads) index_scores_simt(IndexParams p) {
  extern __shared__ float qs[];   // [kQB][n_hI][c_I] then w [kQB][n_hI]
  const int b = blockIdx.z;
  const int q0 = blockIdx.y * kQB;
  const int nq = min(kQB, p.n_q - q0);
  const int HC = p.n_hI * p.c_I;
  float *ws = qs + kQB * HC;
  for (int i = threadIdx.x; i < nq * HC; i += blockDim.x) {
    const Tq *src = reinterpret_cast<const Tq *>(p.qI) + ((long long)b * p.n_q + q0) * HC;
    qs[i] = Elt<Tq>::load(src + i);
  }
  for (int i = threadIdx.x; i < nq * p.n_hI; i += blockDim.x)
    ws[i] = p.wI[((long long)b * p.n_q + q0) * p.n_hI + i];
  __syncthreads();
  const long long s = (long long)blockIdx.x * kScoreThreads + threadIdx.x;
  const int Vlast = (p.start_pos + q0 + nq) / p.m;   // entries visible to the last query
  if (s >= Vlast) return;
  float kscale = 1.f;
  if (p.key_dtype == HCA_FP8E4M3) kscale = p.KI_scale[(long long)b * p.cap + s];
  float acc[kQB];
#pragma unroll
  for (int j = 0; j < kQB; ++j) acc[j] = 0.f;
  for (int h = 0; h < p.n_hI; ++h) {
    float dot[kQB];
#pragma unroll
    for (int j = 0; j < kQB; ++j) dot[j] = 0.f;
    for (int d = 0; d < p.c_I; ++d) {
      float kv;
      if (p.key_dtype == HCA_FP8E4M3) {
        const uint8_t byte = reinterpret_cast<const uint8_t *>(p.KI)[((long long)b * p.cap + s) * p.c_I + d];
        __half_raw hr = __nv_cvt_fp8_to_halfraw(byte, __NV_E4M3);
        kv = __half2float(__half(hr));
      } else {
        kv = Elt<Tk>::load(reinterpret_cast<const Tk *>(p.KI) + ((long long)b * p.cap + s) * p.c_I + d);
      }
#pragma unroll
      for (int j = 0; j < kQB; ++j) dot[j] += qs[(j * p.n_hI + h) * p.c_I + d] * kv;
    }
#pragma unroll
    for (int j = 0; j < kQB; ++j) acc[j] += ws[j * p.n_hI + h] * fmaxf(dot[j], 0.f);
  }
  for (int j = 0; j < nq; ++j) {
    const int t = p.start_pos + q0 + j;
    float v = acc[j] * kscale;
    if (p.round_bf16) v = __bfloat162float(__float2bfloat16_rn(v));
    if (s < (t + 1) / p.m) p.scores[((long long)b * p.n_q + q0 + j) * p.score_stride + s] = v;
  }
}

// ------------------------------------------------------------------ top-k
// One thread-block cluster of C CTAs (C <= 8) selects the top-k of one row
// segment; CTA r of the cluster holds keys [r*slice, (r+1)*slice) of the
// segment in shared memory.  The radix select takes three digits of the
// order key: bits 31..21 (2048 bins), 20..10 (2048 bins) and 9..0.  The wide
// first digit already separates scores of one binade, so after it only the
// keys of the threshold's bin (compacted into kCandMax slots when they fit)
// take part in the later passes.  With C > 1 every CTA adds its non-empty
// bins into every CTA's copy of the cluster histogram with distributed-
// shared-memory atomics (double-buffered by pass parity), so that after one
// cluster barrier each CTA derives the same digit on its own.  The final stable compaction offsets each CTA's output by the
// winners of the lower-ranked CTAs, so the selection leaves in ascending
// index order with ties resolved towards the lower index.  Rows longer than
// one segment are cut into segments whose winners (order key + index) a
// second launch merges.
// selection kernel: 0 = by shape, 1 = a CTA per row, 2 = a warp per row,
// 3 = the segmented cluster select, 4 = a cluster per row (hca_topk_kernel)
int g_topk_kernel = 0;
constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kSliceMax = 16384;   // keys per CTA (64 KB of shared memory)
constexpr int kCandMax = 2048;     // compacted keys per CTA (8 KB)
constexpr int kClusterMax = 8;     // portable cluster size
constexpr int kBinsMax = 2048;
constexpr uint32_t kNoBin = 0xFFFFFFFFu;
// digit p covers bits [shift, shift + width)
__device__ __forceinline__ int digit_shift(int pass) { return pass == 0 ? 21 : (pass == 1 ? 10 : 0); }
__device__ __forceinline__ int digit_width(int pass) { return pass == 2 ? 10 : 11; }

// The float of an order key (inverse of order_bits; -0 comes back as +0).
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ uint32_t order_bits(uint32_t u) {
  if ((u & 0x7FFFFFFFu) == 0) u = 0;                 // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // >= 1 for every non-NaN float
}
// Copy len 32-bit words to shared memory, as order keys (KEYS: already keys).
template <bool KEYS>
__device__ __forceinline__ void load_keys(uint32_t *dst, const uint32_t *src, int len) {
  const int tid = threadIdx.x;
  int done = 0;
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    const int nv = len >> 2;
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    for (int i0 = 0; i0 < nv; i0 += 4 * kTopkThreads) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = i0 + u * kTopkThreads + tid;
        if (j < nv) v[u] = __ldg(s4 + j);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = i0 + u * kTopkThreads + tid;
        if (j < nv) {
          uint4 x = v[u];
          if (!KEYS) { x.x = order_bits(x.x); x.y = order_bits(x.y); x.z = order_bits(x.z); x.w = order_bits(x.w); }
          d4[j] = x;
        }
      }
    }
    done = nv * 4;
  }
  for (int i = done + tid; i < len; i += kTopkThreads) {
    const uint32_t x = __ldg(src + i);
    dst[i] = KEYS ? x : order_bits(x);
  }
}

// Over the histogram h[0..nb) taken from the top bin down: the bin in which
// the krem-th largest key falls, krem within that bin, and the histogram's
// total.  All threads call; results land in out[0..2] (digit, krem, total).
__device__ void find_digit(const uint32_t *h, int nb, int krem, int *warp_tot, int *out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (nb + kTopkThreads - 1) / kTopkThreads;
  const int hi = nb - 1 - tid * per;                       // this thread's bins: hi, hi-1, ..., > hi-per
  int sum = 0;
  for (int j = 0; j < per; ++j)
    if (hi - j >= 0) sum += (int)h[hi - j];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = lane < kTopkWarps ? warp_tot[lane] : 0;
    int u = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, u, o);
      if (lane >= o) u += y;
    }
    if (lane < kTopkWarps) warp_tot[lane] = u - t;          // exclusive warp offsets
    if (lane == kTopkWarps - 1) out[2] = u;                  // total
  }
  __syncthreads();
  int above = warp_tot[warp] + incl - sum;                   // keys in higher bins than this thread's
  if (above < krem && above + sum >= krem) {
    for (int j = 0; j < per; ++j) {
      const int b = hi - j;
      if (b < 0) break;
      const int c = (int)h[b];
      if (above + c >= krem) {
        out[0] = b;
        out[1] = krem - above;
        break;
      }
      above += c;
    }
  }
  __syncthreads();
}

// Grid: x = C * rows * n_seg, cluster (C,1,1).  Dynamic shared memory:
// (slice + kCandMax) words.
__global__ void __launch_bounds__(kTopkThreads) topk_cluster(TopkParams p) {
  extern __shared__ __align__(16) uint32_t dyn[];
  uint32_t *keys = dyn;               // [slice]
  uint32_t *cand = dyn + p.slice;     // [kCandMax]
  __shared__ __align__(16) uint32_t hist[kBinsMax];       // this CTA's histogram
  __shared__ __align__(16) uint32_t total[2][kBinsMax];   // the cluster's histogram, by pass parity
  __shared__ int warp_tot[32];
  __shared__ __align__(16) int res[4];                 // digit, krem, total of the current pass
  __shared__ __align__(8) int peer_cnt[kClusterMax][2];   // every CTA's keys above / equal to the threshold
  __shared__ int w_gt[kTopkWarps], w_eq[kTopkWarps];
  __shared__ int s_nc, s_base, s_eqb;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t C = cluster_nctarank(), rank = cluster_ctarank();
  const long long unit = blockIdx.x / C;
  const int row = (int)(unit / p.n_seg), seg = (int)(unit % p.n_seg);
  const int V = p.fixed_len > 0 ? p.fixed_len : (p.start_pos + row % p.n_q + 1) / p.m;
  const long long seg_begin = (long long)seg * p.seg_len;
  const int seg_V = (int)max(0LL, min((long long)p.seg_len, (long long)V - seg_begin));
  const int len = max(0, min(p.slice, seg_V - (int)rank * p.slice));
  const long long begin = seg_begin + (long long)rank * p.slice;   // element index of keys[0]

  const unsigned long long st_entry = global_ns();
  pdl_trigger();   // the attention may start its prologue
  pdl_wait();      // the scores of the previous launch are complete
  const unsigned long long st_ready = global_ns();
  if (p.keys) load_keys<true>(keys, p.keys + row * p.in_stride + begin, len);
  else load_keys<false>(keys, reinterpret_cast<const uint32_t *>(p.scores) + row * p.in_stride + begin, len);
  for (int i = tid; i < kBinsMax; i += kTopkThreads) {
    hist[i] = 0;
    total[0][i] = 0;
    total[1][i] = 0;
  }
  if (tid == 0) s_nc = 0;
  if (C > 1) cluster_sync();   // every CTA's totals are clear before anyone adds into them
  else __syncthreads();

  uint32_t prefix = 0, mask = 0, T = 0;
  int krem = p.k, K = 0;
  bool compacted = false;
  int nc = 0;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = digit_shift(pass), nb = 1 << digit_width(pass);
    const uint32_t *arr = compacted ? cand : keys;
    const int n = compacted ? nc : len;
    for (int b0 = 0; b0 < n; b0 += kTopkThreads) {
      const int i = b0 + tid;
      uint32_t bin = kNoBin;
      if (i < n) {
        const uint32_t kk = arr[i];
        if (kk != 0 && (kk & mask) == prefix) bin = (kk >> shift) & (uint32_t)(nb - 1);
      }
      if (bin != kNoBin) atomicAdd(&hist[bin], 1u);
    }
    __syncthreads();
    if (C > 1) {
      // add this CTA's non-empty bins into every CTA's total of this pass; a
      // total is cleared two passes before it is reused, with a cluster
      // barrier in between
      uint32_t *tp = total[pass & 1];
      const uint32_t t0 = smem_u32(tp);
      for (int b = tid; b < nb; b += kTopkThreads) {
        const uint32_t c = hist[b];
        if (c)
          for (uint32_t r = 0; r < C; ++r)
            asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(cluster_map(t0 + 4u * b, r)), "r"(c)
                         : "memory");
      }
      cluster_sync();
      find_digit(tp, nb, krem, warp_tot, res);
      for (int b = tid; b < nb; b += kTopkThreads) tp[b] = 0;
    } else {
      find_digit(hist, nb, krem, warp_tot, res);
    }
    if (pass == 0) {
      const int nvalid = res[2];   // the whole segment's keys (absent keys are 0)
      if (nvalid <= p.k) { K = nvalid; krem = 0; break; }   // every key is selected, T = 0
      if (p.k <= 0) { K = 0; krem = 0; prefix = 0xFFFFFFFFu; break; }   // none is selected
      K = p.k;
    }
    const uint32_t digit = (uint32_t)res[0];
    prefix |= digit << shift;
    mask |= (uint32_t)(nb - 1) << shift;
    krem = res[1];
    const uint32_t local_in_bin = hist[digit];
    if (pass < 2 && !compacted && local_in_bin <= (uint32_t)kCandMax) {
      // compact this CTA's keys that match the new prefix
      for (int b0 = 0; b0 < n; b0 += kTopkThreads) {
        const int i = b0 + tid;
        const uint32_t kk = i < n ? arr[i] : 0u;
        const bool m = kk != 0 && (kk & mask) == prefix;
        const unsigned bal = __ballot_sync(0xffffffffu, m);
        int at = 0;
        if (lane == 0 && bal) at = atomicAdd(&s_nc, __popc(bal));
        at = __shfl_sync(0xffffffffu, at, 0) + __popc(bal & ((1u << lane) - 1u));
        if (m) cand[at] = kk;
      }
      nc = (int)local_in_bin;
      compacted = true;
    }
    __syncthreads();   // every thread has read hist[digit]
    for (int b = tid; b < nb; b += kTopkThreads) hist[b] = 0;
    __syncthreads();
  }
  if (K == p.k) T = prefix;

  // count, per warp over a contiguous run of keys, those above and equal to T
  const int wseg = ((len + kTopkThreads - 1) / kTopkThreads) * 32;
  const int w_lo = min(len, warp * wseg), w_hi = min(len, w_lo + wseg);
  int gt = 0, eq = 0;
  for (int i0 = w_lo; i0 < w_hi; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t kk = i < w_hi ? keys[i] : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, kk > T));
    eq += __popc(__ballot_sync(0xffffffffu, T != 0 && kk == T));
  }
  if (lane == 0) { w_gt[warp] = gt; w_eq[warp] = eq; }
  __syncthreads();
  if (tid == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < kTopkWarps; ++w) { a += w_gt[w]; b += w_eq[w]; }
    const uint32_t at = smem_u32(&peer_cnt[rank][0]);
    for (uint32_t r = 0; r < C; ++r) st_dsmem_u32x2(cluster_map(at, r), (uint32_t)a, (uint32_t)b);
  }
  // every CTA's counts have landed; no CTA touches another's shared memory after this
  if (C > 1) cluster_sync();
  else __syncthreads();
  if (tid == 0) {
    // winners of the lower-ranked CTAs, and ties among them
    int base = 0, eqb = 0;
    for (uint32_t r = 0; r < rank; ++r) {
      base += peer_cnt[r][0] + max(0, min(krem - eqb, peer_cnt[r][1]));
      eqb += peer_cnt[r][1];
    }
    s_base = base;
    s_eqb = eqb;
  }
  __syncthreads();
  int ties_before = s_eqb, sel_before = s_base;
  for (int w = 0; w < warp; ++w) { ties_before += w_eq[w]; sel_before += w_gt[w]; }
  sel_before += min(krem, ties_before) - min(krem, s_eqb);
  int32_t *out = p.idx_out + row * p.out_stride + (long long)seg * p.k;
  uint32_t *kout = p.key_out ? p.key_out + row * p.out_stride + (long long)seg * p.k : nullptr;
  const int32_t *cidx = p.cand_idx ? p.cand_idx + row * p.in_stride + begin : nullptr;
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = w_lo; i0 < w_hi; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t kk = i < w_hi ? keys[i] : 0u;
    const bool is_eq = T != 0 && kk == T;
    const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
    const bool take = kk > T || (is_eq && ties_before + __popc(eqm & lt) < krem);
    const unsigned sm = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int o = sel_before + __popc(sm & lt);
      out[o] = cidx ? cidx[i] : (int32_t)(begin + i);
      if (kout) kout[o] = kk;
    }
    ties_before += __popc(eqm);
    sel_before += __popc(sm);
  }
  if (rank == 0)
    for (int i = K + tid; i < p.k; i += kTopkThreads) {
      out[i] = -1;
      if (kout) kout[i] = 0u;
    }
  if (step_trace_on()) {
    __syncthreads();
    if (tid == 0) step_trace_record(ST_TOPK, st_entry, st_ready);
  }
}

// ------------------------------------------------------------ one CTA per row
// Rows of up to 32 * NT keys: one CTA holds the whole row in registers (eight
// 16-byte loads per thread, all in flight at once) and selects in one pass:
//   1. a sample of the row (one key per thread, spread over the whole row)
//      gives two thresholds t_hi > t_lo between which the k-th largest score
//      falls with high probability (sample ranks of about k*S/V -+ 3 sigma);
//   2. every key is compared with them: keys above t_hi are marked as winners
//      in a bit mask of the row, keys in [t_lo, t_hi] are compacted into a
//      band list (a few times k keys);
//   3. if the counts confirm that the k-th score lies in the band, an exact
//      radix select over the band's order keys finds the threshold key T and
//      the number of ties at T to keep; otherwise (ties or an unlucky sample)
//      the same exact select runs over the whole row held in registers;
//   4. the winners' and the kept ties' bits are emitted in ascending index
//      order (ties to the lower index) by a block scan over the mask words.
// Every decision is exact: the thresholds only decide how much of the row the
// exact select has to look at.
constexpr int kRowRegs = 8;        // 16-byte loads per thread: rows of up to 32 * NT keys
constexpr int kRowMaxNT = 1024;
constexpr int kRowMax = 32 * kRowMaxNT;
constexpr int kRowCand = 4096;     // band keys held in shared memory (order key + index)
constexpr int kRowSample = 1024;   // at most one sample key per thread

template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_buf, int *total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = lane < NW ? warp_buf[lane] : 0;
    int u = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, u, o);
      if (lane >= o) u += y;
    }
    if (lane < NW) warp_buf[lane] = u - t;
    if (lane == NW - 1) *total = u;
  }
  __syncthreads();
  const int r = warp_buf[warp] + incl - v;
  __syncthreads();   // warp_buf may be reused by the caller
  return r;
}

// The bin (counted from the top) of the krem-th largest element of histogram
// h[0..nb), and krem within that bin: out[0] = bin, out[1] = krem in bin.
template <int NT>
__device__ __forceinline__ void row_find_digit(const uint32_t *h, int nb, int krem, int *warp_buf, int *scan_tot,
                                               int *out) {
  const int per = (nb + NT - 1) / NT;
  const int hi = nb - 1 - (int)threadIdx.x * per;   // this thread's bins hi, hi-1, ..., > hi-per
  int sum = 0;
  for (int j = 0; j < per; ++j)
    if (hi - j >= 0) sum += (int)h[hi - j];
  int above = block_exclusive_scan<NT>(sum, warp_buf, scan_tot);
  if (above < krem && above + sum >= krem) {
    for (int j = 0; j < per; ++j) {
      const int b = hi - j;
      if (b < 0) break;
      const int c = (int)h[b];
      if (above + c >= krem) {
        out[0] = b;
        out[1] = krem - above;
        break;
      }
      above += c;
    }
  }
  __syncthreads();
}

// Shared state of one row's selection.
struct RowSel {
  uint32_t hist[kBinsMax];
  int warp_buf[32];
  int res[2];
  int scan_tot;
  int s_above, s_nc;
  uint32_t s_min, s_max;
};

// Exact radix select of the krem-th largest order key among a set of keys
// that each(f) visits (every thread calls f on its share of the keys; 0 =
// no key).  Distances from kmin are taken in digits of up to 11 bits from
// their highest differing bit.  Returns T (the key) and, in *krem, how many
// keys equal to T are kept.
template <int NT, typename Each>
__device__ uint32_t radix_select(RowSel &sh, uint32_t kmin, uint32_t kmax, int *krem, Each each) {
  const int tid = threadIdx.x;
  const uint32_t range = kmax - kmin;
  const int nbits = range ? 32 - __clz(range) : 0;
  uint32_t prefix = 0;
  int shift = nbits;
  while (shift > 0) {
    const int width = shift > 11 ? 11 : shift;
    const int nshift = shift - width;
    const int nb = 1 << width;
    each([&](uint32_t kk) {
      if (kk == 0 || kk < kmin || kk > kmax) return;
      const uint32_t v = kk - kmin;
      if (shift >= 32 || (v >> shift) == prefix) atomicAdd(&sh.hist[(v >> nshift) & (uint32_t)(nb - 1)], 1u);
    });
    __syncthreads();
    row_find_digit<NT>(sh.hist, nb, *krem, sh.warp_buf, &sh.scan_tot, sh.res);
    const uint32_t digit = (uint32_t)sh.res[0];
    *krem = sh.res[1];
    __syncthreads();   // every thread has read res
    for (int i = tid; i < nb; i += NT) sh.hist[i] = 0;
    __syncthreads();
    prefix = (prefix << width) | digit;
    shift = nshift;
  }
  return kmin + prefix;
}

// Grid: one CTA per row.  Dynamic shared memory: 2 * words + 2 * kRowCand
// words (winner and tie masks of the row, band keys and indices).
template <int NT, int RR>
__global__ void __launch_bounds__(NT) topk_row(TopkParams p) {
  constexpr int NW = NT / 32;
  extern __shared__ __align__(16) uint32_t dyn[];
  __shared__ RowSel sh;
  __shared__ uint32_t red_a[NW], red_b[NW];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  const int V = p.fixed_len > 0 ? p.fixed_len : (p.start_pos + row % p.n_q + 1) / p.m;
  const int nwords = (V + 31) >> 5;
  uint32_t *win = dyn;                        // [nwords_max]
  uint32_t *tie = dyn + p.slice;              // [nwords_max]
  uint32_t *band_key = dyn + 2 * p.slice;     // [kRowCand]
  uint32_t *band_idx = band_key + kRowCand;   // [kRowCand]
  int32_t *out = p.idx_out + (long long)row * p.out_stride;
  const unsigned long long st_entry = global_ns();
  pdl_trigger();   // the attention may start its prologue
  pdl_wait();      // the scores of the previous launch are complete
  const unsigned long long st_ready = global_ns();
  if (p.k <= 0) return;

  // ---- the row in registers: thread t holds keys 4t + 4NT*j + e (as floats)
  const float *src = p.scores + (long long)row * p.in_stride;
  float x[RR][4];
  const bool vec = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
#pragma unroll
  for (int j = 0; j < RR; ++j) {
    const int i = 4 * tid + 4 * NT * j;
    if (vec && i + 3 < V) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(src + i));
      x[j][0] = v.x; x[j][1] = v.y; x[j][2] = v.z; x[j][3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) x[j][e] = i + e < V ? __ldg(src + i + e) : 0.f;
    }
  }
  for (int w = tid; w < nwords; w += NT) { win[w] = 0u; tie[w] = 0u; }
  for (int i = tid; i < kBinsMax; i += NT) sh.hist[i] = 0u;
  if (tid == 0) { sh.s_above = 0; sh.s_nc = 0; }

  int krem = 0;        // ties at T to keep
  uint32_t T = 0;      // the k-th largest order key (0: every key is kept)
  bool banded = false;
  if (V > p.k) {
    // ---- 1. sample: thread t contributes key 4t + 4NT*(t % 8) (its register j = t % 8)
    const int js = tid % RR;
    const int is = 4 * tid + 4 * NT * js;
    const bool has_s = is < V && tid < kRowSample;
    float sv = 0.f;
#pragma unroll
    for (int j = 0; j < RR; ++j)
      if (j == js) sv = x[j][0];
    uint32_t smin = has_s ? order_bits(__float_as_uint(sv)) : 0xFFFFFFFFu;
    uint32_t smax = has_s ? smin : 0u;
    int ns = has_s ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      smin = min(smin, __shfl_xor_sync(0xffffffffu, smin, o));
      smax = max(smax, __shfl_xor_sync(0xffffffffu, smax, o));
      ns += __shfl_xor_sync(0xffffffffu, ns, o);
    }
    if (lane == 0) { red_a[warp] = smin; red_b[warp] = smax; sh.warp_buf[warp] = ns; }
    __syncthreads();
    smin = red_a[0]; smax = red_b[0]; ns = sh.warp_buf[0];
    for (int w = 1; w < NW; ++w) { smin = min(smin, red_a[w]); smax = max(smax, red_b[w]); ns += sh.warp_buf[w]; }
    __syncthreads();
    const float lo = key_float(smin), hi = key_float(smax);
    const float scale = (float)kBinsMax / (hi - lo);
    if (ns >= 64 && smin != smax && scale > 0.f && scale < INFINITY) {
      // 2048 equal-width bins of the sample values; ranks from the top
      if (has_s) {
        const float f = (key_float(order_bits(__float_as_uint(sv))) - lo) * scale;
        const uint32_t b = f >= (float)(kBinsMax - 1) ? (uint32_t)(kBinsMax - 1) : (f > 0.f ? (uint32_t)f : 0u);
        atomicAdd(&sh.hist[b], 1u);
      }
      __syncthreads();
      const float q = (float)p.k * (float)ns / (float)V;   // sample keys expected above the k-th
      const int r_hi = max(1, (int)floorf(q - 3.f * sqrtf(q)));
      const int r_lo = min(ns, (int)ceilf(q + 3.f * sqrtf(q) + 2.f));
      row_find_digit<NT>(sh.hist, kBinsMax, r_hi, sh.warp_buf, &sh.scan_tot, sh.res);
      const int b_hi = sh.res[0];
      __syncthreads();
      row_find_digit<NT>(sh.hist, kBinsMax, r_lo, sh.warp_buf, &sh.scan_tot, sh.res);
      const int b_lo = sh.res[0];
      __syncthreads();
      for (int i = tid; i < kBinsMax; i += NT) sh.hist[i] = 0u;
      // thresholds at the bin edges: above t_hi = winners, [t_lo, t_hi] = band
      const float t_hi = lo + (float)(b_hi + 1) / scale;
      const float t_lo = lo + (float)b_lo / scale;
      // ---- 2. one pass over the row: count, then place (no per-key votes)
      int above = 0, inband = 0;
#pragma unroll
      for (int j = 0; j < RR; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool valid = 4 * tid + 4 * NT * j + e < V;
          const float v = x[j][e];
          above += (valid && v > t_hi) ? 1 : 0;
          inband += (valid && v <= t_hi && v >= t_lo) ? 1 : 0;
        }
      // band slots: warp-inclusive scan of the per-thread counts, one atomic per warp
      int incl = inband;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int wbase = 0;
      if (lane == 31 && incl) wbase = atomicAdd(&sh.s_nc, incl);
      int at = __shfl_sync(0xffffffffu, wbase, 31) + incl - inband;
      if (above | inband) {
#pragma unroll
        for (int j = 0; j < RR; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * tid + 4 * NT * j + e;
            const float v = x[j][e];
            if (i < V && v > t_hi) {
              atomicOr(&win[i >> 5], 1u << (i & 31));
            } else if (i < V && v >= t_lo) {
              if (at < kRowCand) {
                band_key[at] = order_bits(__float_as_uint(v));
                band_idx[at] = (uint32_t)i;
              }
              ++at;
            }
          }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
      if (lane == 0) atomicAdd(&sh.s_above, above);
      __syncthreads();
      const int na = sh.s_above, nc = sh.s_nc;
      banded = na < p.k && na + nc >= p.k && nc <= kRowCand;
      if (banded) {
        // ---- 3. exact select within the band
        uint32_t cmin = 0xFFFFFFFFu, cmax = 0u;
        for (int i = tid; i < nc; i += NT) { cmin = min(cmin, band_key[i]); cmax = max(cmax, band_key[i]); }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          cmin = min(cmin, __shfl_xor_sync(0xffffffffu, cmin, o));
          cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
        }
        if (lane == 0) { red_a[warp] = cmin; red_b[warp] = cmax; }
        __syncthreads();
        cmin = red_a[0]; cmax = red_b[0];
        for (int w = 1; w < NW; ++w) { cmin = min(cmin, red_a[w]); cmax = max(cmax, red_b[w]); }
        krem = p.k - na;
        T = radix_select<NT>(sh, cmin, cmax, &krem, [&](auto f) {
          for (int i = tid; i < nc; i += NT) f(band_key[i]);
        });
        for (int i = tid; i < nc; i += NT) {
          const uint32_t kk = band_key[i], ix = band_idx[i];
          if (kk > T) atomicOr(&win[ix >> 5], 1u << (ix & 31));
          else if (kk == T) atomicOr(&tie[ix >> 5], 1u << (ix & 31));
        }
      } else {
        // the band missed the k-th score: clear the winner marks
        for (int w = tid; w < nwords; w += NT) win[w] = 0u;
      }
      __syncthreads();
    }
    if (!banded) {
      // ---- 3'. exact select over the whole row (registers)
      uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
      for (int j = 0; j < RR; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * tid + 4 * NT * j + e < V) {
            const uint32_t kk = order_bits(__float_as_uint(x[j][e]));
            kmin = min(kmin, kk);
            kmax = max(kmax, kk);
          }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      }
      if (lane == 0) { red_a[warp] = kmin; red_b[warp] = kmax; }
      __syncthreads();
      kmin = red_a[0]; kmax = red_b[0];
      for (int w = 1; w < NW; ++w) { kmin = min(kmin, red_a[w]); kmax = max(kmax, red_b[w]); }
      krem = p.k;
      T = radix_select<NT>(sh, kmin, kmax, &krem, [&](auto f) {
#pragma unroll
        for (int j = 0; j < RR; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (4 * tid + 4 * NT * j + e < V) f(order_bits(__float_as_uint(x[j][e])));
      });
#pragma unroll
      for (int j = 0; j < RR; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * tid + 4 * NT * j + e;
          if (i < V) {
            const uint32_t kk = order_bits(__float_as_uint(x[j][e]));
            if (kk > T) atomicOr(&win[i >> 5], 1u << (i & 31));
            else if (kk == T) atomicOr(&tie[i >> 5], 1u << (i & 31));
          }
        }
      __syncthreads();
    }
  } else {
    // every key is kept
    for (int w = tid; w < nwords; w += NT) win[w] = (w < (V >> 5)) ? 0xFFFFFFFFu : ((1u << (V & 31)) - 1u);
    __syncthreads();
  }

  // ---- 4. emit the winners and the first krem ties in ascending index order
  constexpr int kWordsPerThread = (kRowMax / 32 + NT - 1) / NT;
  const int wpt = (nwords + NT - 1) / NT;
  const int w0 = tid * wpt;
  int my_ties = 0;
  for (int u = 0; u < wpt && u < kWordsPerThread; ++u)
    if (w0 + u < nwords) my_ties += __popc(tie[w0 + u]);
  int ties_before = block_exclusive_scan<NT>(my_ties, sh.warp_buf, &sh.scan_tot);
  int my_sel = 0;
  {
    int tb = ties_before;
    for (int u = 0; u < wpt && u < kWordsPerThread; ++u)
      if (w0 + u < nwords) {
        const int nt = __popc(tie[w0 + u]);
        my_sel += __popc(win[w0 + u]) + max(0, min(nt, krem - tb));
        tb += nt;
      }
  }
  int at = block_exclusive_scan<NT>(my_sel, sh.warp_buf, &sh.scan_tot);
  for (int u = 0; u < wpt && u < kWordsPerThread; ++u) {
    const int w = w0 + u;
    if (w >= nwords) break;
    uint32_t wm = win[w], tm = tie[w];
    while (wm | tm) {
      const int bw = wm ? __ffs(wm) - 1 : 32, bt = tm ? __ffs(tm) - 1 : 32;
      if (bw < bt) {
        out[at++] = w * 32 + bw;
        wm &= wm - 1u;
      } else {
        if (ties_before < krem) out[at++] = w * 32 + bt;
        ++ties_before;
        tm &= tm - 1u;
      }
    }
  }
  const int K = V < p.k ? V : p.k;
  for (int i = K + tid; i < p.k; i += NT) out[i] = -1;
  if (step_trace_on()) {
    __syncthreads();
    if (tid == 0) step_trace_record(ST_TOPK, st_entry, st_ready);
  }
}

// ------------------------------------------------------- a warp per row
// Many rows (prefill): each warp of a CTA selects one row, with no block-wide
// barrier, so that many rows are in flight per SM and the pass over the
// scores runs at the memory rate.  Per row:
//   1. a sample of the row (32 to 128 evenly spaced runs of 8 keys, one
//      32-byte sector each; the whole row when it has at most 1024 keys) gives, by
//      radix select over the sample, two thresholds: keys above hiK are
//      winners, keys in [loK, hiK] are the band, which holds the k-th largest
//      unless the sample misled (then step 3's fallback decides);
//   2. one pass over the row (128 consecutive keys per warp step, 4 per lane,
//      8 steps' loads in flight): winners go to a bit mask of the row, band keys (order
//      key + index) to a list in shared memory in ascending index order;
//   3. if the winners number below k and winners + band reach k (and the band
//      fitted its list), an exact radix select over the band finds the k-th
//      largest key T and how many keys equal to T are kept (krem); the band's
//      keys above T and its first krem keys equal to T (lowest indices) join
//      the mask.  Otherwise (rare) counting passes over the row narrow the
//      range that holds the k-th largest, 256 bins at a time, until its bin
//      fits the band list (the band pass then runs again on that bin) or is a
//      single key value (a last pass marks the keys above it and its first
//      ties);
//   4. the mask's bits are emitted in ascending index order.
// Every decision is exact; the sample only decides how much of the row the
// exact select looks at.
constexpr int kWarpRowWarps = 8;                 // warps (rows) per CTA
constexpr int kWarpRowMaxWords = kRowMax / 32;   // mask words of the longest row
constexpr int kWarpRowCand = 1536;               // band keys held per warp
constexpr int kWarpRowSample = 1024;             // sample keys per row (32 per lane)
constexpr int kWarpRowUnroll = 8;                // steps whose loads are in flight together
// 13 KB per warp: two CTAs of 8 warps fit an SM
struct WarpRowSmem {
  uint32_t mask[kWarpRowMaxWords];
  uint32_t cand_key[kWarpRowCand];
  uint16_t cand_idx[kWarpRowCand];   // indices < kRowMax = 32768
};
static_assert(kRowMax <= 65536, "band indices are 16-bit");
static_assert(kWarpRowSample <= kWarpRowCand, "the sample is held in the band list");

// Exact radix select (digits of up to 8 bits from the highest bit in which
// kmin and kmax differ) of the krem-th largest key among those each(f)
// visits (every lane calls f on its share), with a 256-bin histogram in
// shared memory.  Returns the key; *krem becomes how many keys equal to it
// are kept.
template <typename Each>
__device__ uint32_t warp_radix_select(uint32_t *hist, uint32_t kmin, uint32_t kmax, int *krem, Each each) {
  const int lane = threadIdx.x & 31;
  const uint32_t range = kmax - kmin;
  int shift = range ? 32 - __clz(range) : 0;
  uint32_t prefix = 0;
  while (shift > 0) {
    const int width = shift > 8 ? 8 : shift;
    const int nshift = shift - width;
    for (int i = lane; i < 256; i += 32) hist[i] = 0u;
    __syncwarp();
    each([&](uint32_t kk) {
      if (kk < kmin || kk > kmax) return;
      const uint32_t v = kk - kmin;
      if (shift >= 32 || (v >> shift) == prefix) atomicAdd(&hist[(v >> nshift) & ((1u << width) - 1u)], 1u);
    });
    __syncwarp();
    // lane l holds bins 255-8l .. 248-8l (from the top); counts above each lane's bins
    uint32_t h[8];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      h[j] = hist[255 - 8 * lane - j];
      sum += (int)h[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int above = incl - sum;
    int found = -1, kin = 0;
    if (above < *krem && incl >= *krem) {
      int a = above;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (found < 0 && a + (int)h[j] >= *krem) {
          found = 255 - 8 * lane - j;
          kin = *krem - a;
        }
        a += (int)h[j];
      }
    }
    const unsigned who = __ballot_sync(0xffffffffu, found >= 0);
    const int src = __ffs(who) - 1;
    const int digit = __shfl_sync(0xffffffffu, found, src);
    *krem = __shfl_sync(0xffffffffu, kin, src);
    prefix = (prefix << width) | (uint32_t)digit;
    shift = nshift;
    __syncwarp();
  }
  return kmin + prefix;
}

__global__ void __launch_bounds__(kWarpRowWarps * 32) topk_warp(TopkParams p) {
  extern __shared__ __align__(16) uint8_t dyn_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  WarpRowSmem &sm = reinterpret_cast<WarpRowSmem *>(dyn_raw)[warp];
  __shared__ uint32_t hist_all[kWarpRowWarps][256];
  uint32_t *hist = hist_all[warp];
  const long long row = (long long)blockIdx.x * kWarpRowWarps + warp;
  const unsigned long long st_entry = global_ns();
  pdl_trigger();   // the attention may start its prologue
  pdl_wait();      // the scores of the previous launch are complete
  const unsigned long long st_ready = global_ns();
  if (row >= p.rows || p.k <= 0) return;
  const int V = p.fixed_len > 0 ? p.fixed_len : (p.start_pos + (int)(row % p.n_q) + 1) / p.m;
  const int k = p.k;
  int32_t *out = p.idx_out + row * p.out_stride;
  const float *src = p.scores + row * p.in_stride;
  const uint32_t *srcu = reinterpret_cast<const uint32_t *>(src);
  const int nwords = (V + 31) >> 5;
  if (V <= k) {
    for (int i = lane; i < k; i += 32) out[i] = i < V ? i : -1;
    return;
  }
  const uint32_t lt = (1u << lane) - 1u;
  const int steps = (V + 127) >> 7;
  // One pass over the row in batches of 8 steps of 128 keys: f(st0, v) with
  // v[u][e] = key 128 (st0 + u) + 32 e + lane (-inf past the row); a batch's
  // loads are all in flight together and the next batch's lines are
  // prefetched to L2.
  auto scan_row = [&](auto f) {
#pragma unroll 1
    for (int st0 = 0; st0 < steps; st0 += kWarpRowUnroll) {
      float v[kWarpRowUnroll][4];
#pragma unroll
      for (int u = 0; u < kWarpRowUnroll; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = (st0 + u) * 128 + 32 * e + lane;
          v[u][e] = i < V ? __ldg(src + i) : -INFINITY;
        }
      {
        const int i = (st0 + kWarpRowUnroll) * 128 + 32 * lane;
        if (i < V) asm volatile("prefetch.global.L2 [%0];" ::"l"(src + i));
      }
      f(st0, v);
    }
  };

  // ---- 1. sample (order keys into the band list, which is free until step
  // 2) and thresholds: the r_hi-th and r_lo-th largest sample keys, by radix
  // select over the sample
  // S scales with k V so that the band holds ~800 keys whatever the row length
  // (q = k S / V stays near k^2 / 16384): 256, 512 or 1024 sample keys
  const long long kv = (long long)k * V;
  const int S = V <= kWarpRowSample ? V : (kv <= (4ll << 20) ? 256 : (kv <= (8ll << 20) ? 512 : 1024));
  if (V <= kWarpRowSample) {
    for (int i = lane; i < S; i += 32) sm.cand_key[i] = order_bits(__ldg(srcu + i));
  } else {
    // S/8 runs of 8 keys, R = S/256 per lane; run j starts at the multiple of
    // 8 at or below (2j+1) V / (S/4), kept inside the row
    const int R = S >> 8;
    uint32_t sv[32];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (r < R) {
        const int j = R * lane + r;
        const int st = min(V - 8, (int)(((long long)(2 * j + 1) * V * 4) / S) & ~7);
#pragma unroll
        for (int e = 0; e < 8; ++e) sv[8 * r + e] = __ldg(srcu + st + e);
      }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < 8 * R) sm.cand_key[32 * i + lane] = order_bits(sv[i]);
  }
  __syncwarp();
  uint32_t smin = 0xFFFFFFFFu, smax = 0u;
  for (int i = lane; i < S; i += 32) {
    smin = min(smin, sm.cand_key[i]);
    smax = max(smax, sm.cand_key[i]);
  }
  smin = __reduce_min_sync(0xffffffffu, smin);
  smax = __reduce_max_sync(0xffffffffu, smax);
  auto sample_rank = [&](int r) {
    return warp_radix_select(hist, smin, smax, &r, [&](auto f) {
      for (int i = lane; i < S; i += 32) f(sm.cand_key[i]);
    });
  };
  const float q = (float)k * (float)S / (float)V;   // sample keys expected above the k-th
  const float mg = 3.f * sqrtf(q) + 1.f;
  // winners: keys > hiK (none when the sample's top is within the margin);
  // band: keys in [loK, hiK]
  uint32_t hiK = q - mg >= 1.f ? sample_rank(max(1, (int)floorf(q - mg))) : 0xFFFFFFFFu;
  uint32_t loK = sample_rank(min(S, (int)ceilf(q + mg)));
  __syncwarp();   // the sample is read before the band list is written

  // ---- 2. one pass: winner bits (vote over e = mask word 4 st + e) and the
  // band keys in ascending index order (e first, then lane).  Thresholds
  // compare as floats (the order of non-NaN floats, -0 == +0).
  int nwin = 0, ncand = 0;
  auto band_pass = [&]() {
    // order keys from +inf up (and the NaN images above it) bound nothing
    const float hiF = hiK >= 0xFF800000u ? INFINITY : key_float(hiK), loF = key_float(loK);
    nwin = 0;
    ncand = 0;
    // branch-free over the batch (votes first, then the band appends), so
    // that the steps' work interleaves
    scan_row([&](int st0, const float (&v)[kWarpRowUnroll][4]) {
      uint32_t bc[kWarpRowUnroll][4];
#pragma unroll
      for (int u = 0; u < kWarpRowUnroll; ++u) {
        const int st = st0 + u;
        uint32_t bw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool in = st * 128 + 32 * e + lane < V;
          const bool w = in && v[u][e] > hiF;
          bw[e] = __ballot_sync(0xffffffffu, w);
          bc[u][e] = __ballot_sync(0xffffffffu, in && !w && v[u][e] >= loF);
        }
        if (lane < 4 && st < steps)
          sm.mask[st * 4 + lane] = lane == 0 ? bw[0] : (lane == 1 ? bw[1] : (lane == 2 ? bw[2] : bw[3]));
        nwin += __popc(bw[0]) + __popc(bw[1]) + __popc(bw[2]) + __popc(bw[3]);
      }
#pragma unroll
      for (int u = 0; u < kWarpRowUnroll; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int a = ncand + __popc(bc[u][e] & lt);
          if (((bc[u][e] >> lane) & 1u) && a < kWarpRowCand) {
            sm.cand_key[a] = order_bits(__float_as_uint(v[u][e]));
            sm.cand_idx[a] = (uint16_t)((st0 + u) * 128 + 32 * e + lane);
          }
          ncand += __popc(bc[u][e]);
        }
    });
    __syncwarp();
  };
  band_pass();

  // ---- 2'. the sample misled (rare): narrow exactly.  [lo, hi] holds the
  // k-th largest and `above` keys lie above hi; counting passes split the
  // range into 256 bins (by the top bits of key - lo) until the k-th's bin
  // fits the band list or is a single key value, then the band pass runs on
  // that bin.
  bool tie_class = false;
  if (!(nwin < k && nwin + ncand >= k && ncand <= kWarpRowCand)) {
    uint32_t lo, hi;
    int above;
    if (nwin >= k) { lo = hiK + 1u; hi = 0xFFFFFFFFu; above = 0; }
    else if (nwin + ncand < k) { lo = 0x007FFFFFu; hi = loK - 1u; above = nwin + ncand; }   // from -inf
    else { lo = loK; hi = hiK; above = nwin; }
    for (;;) {
      const uint32_t range = hi - lo;
      const int nb = range ? 32 - __clz(range) : 0;
      if (nb == 0) { tie_class = true; break; }
      const int sh = nb > 8 ? nb - 8 : 0;
      for (int i = lane; i < 256; i += 32) hist[i] = 0u;
      __syncwarp();
      scan_row([&](int st0, const float (&v)[kWarpRowUnroll][4]) {
#pragma unroll
        for (int u = 0; u < kWarpRowUnroll; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t kk = order_bits(__float_as_uint(v[u][e]));
            if ((st0 + u) * 128 + 32 * e + lane < V && kk >= lo && kk <= hi) atomicAdd(&hist[(kk - lo) >> sh], 1u);
          }
      });
      __syncwarp();
      // the bin holding rank k - above (counted from the top)
      int krem = k - above, bin = 0, cnt = 0, acc = 0;
      for (int b = 255; b >= 0; --b) {
        const int c = (int)hist[b];
        if (acc + c >= krem) { bin = b; cnt = c; break; }
        acc += c;
      }
      above += acc;
      const uint32_t nlo = lo + ((uint32_t)bin << sh);
      const uint32_t nhi = (uint32_t)min((unsigned long long)hi, (unsigned long long)nlo + (1ull << sh) - 1ull);
      lo = nlo;
      hi = nhi;
      __syncwarp();
      if (cnt <= kWarpRowCand) break;
    }
    if (tie_class) {
      // every key of [lo, hi] is equal: keys above it, then the first
      // k - above keys equal to it (index order)
      int ties = 0;
      const int krem = k - above;
      scan_row([&](int st0, const float (&v)[kWarpRowUnroll][4]) {
#pragma unroll
        for (int u = 0; u < kWarpRowUnroll; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int st = st0 + u;
            const uint32_t kk = order_bits(__float_as_uint(v[u][e]));
            const bool in = st * 128 + 32 * e + lane < V;
            const bool eq = in && kk == lo;
            const uint32_t be = __ballot_sync(0xffffffffu, eq);
            const bool take = (in && kk > lo) || (eq && ties + __popc(be & lt) < krem);
            const uint32_t word = __ballot_sync(0xffffffffu, take);
            if (lane == e && st < steps) sm.mask[st * 4 + e] = word;
            ties += __popc(be);
          }
      });
      __syncwarp();
    } else {
      hiK = hi;
      loK = lo;
      band_pass();
    }
  }

  // ---- 3. the k-th largest key T within the band and the ties kept: the
  // band's keys above T and its first krem keys equal to T join the mask
  if (!tie_class) {
    uint32_t cmin = 0xFFFFFFFFu, cmax = 0u;
    for (int i = lane; i < ncand; i += 32) {
      cmin = min(cmin, sm.cand_key[i]);
      cmax = max(cmax, sm.cand_key[i]);
    }
    cmin = __reduce_min_sync(0xffffffffu, cmin);
    cmax = __reduce_max_sync(0xffffffffu, cmax);
    int krem = k - nwin;
    const uint32_t T = warp_radix_select(hist, cmin, cmax, &krem, [&](auto f) {
      for (int i = lane; i < ncand; i += 32) f(sm.cand_key[i]);
    });
    int ties = 0;
    for (int c0 = 0; c0 < ncand; c0 += 32) {
      const int i = c0 + lane;
      const uint32_t kk = i < ncand ? sm.cand_key[i] : 0u;
      const bool gt = i < ncand && kk > T, eq = i < ncand && kk == T;
      const uint32_t be = __ballot_sync(0xffffffffu, eq);
      const bool take = gt || (eq && ties + __popc(be & lt) < krem);
      if (take) {
        const uint32_t ix = sm.cand_idx[i];
        atomicOr(&sm.mask[ix >> 5], 1u << (ix & 31));
      }
      ties += __popc(be);
    }
    __syncwarp();
  }

  // ---- 4. emit in ascending index order (exactly k bits are set): lane l
  // takes words [l*wpl, (l+1)*wpl)
  const int wpl = (nwords + 31) >> 5;
  int cnt = 0;
  for (int j = 0; j < wpl; ++j) {
    const int w = lane * wpl + j;
    if (w < nwords) cnt += __popc(sm.mask[w]);
  }
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int at = incl - cnt;
  for (int j = 0; j < wpl; ++j) {
    const int w = lane * wpl + j;
    if (w >= nwords) break;
    uint32_t m = sm.mask[w];
    while (m) {
      const int b = __ffs(m) - 1;
      if (at < k) out[at] = 32 * w + b;
      ++at;
      m &= m - 1u;
    }
  }
  if (step_trace_on() && lane == 0) step_trace_record(ST_TOPK, st_entry, st_ready);
}

// ------------------------------------------------------ a cluster per row
// Few long rows (decode): the row is cut over the C CTAs of a thread-block
// cluster, each holding 32 keys per thread in registers, so that every pass
// over the keys runs on C SMs.  CTA 0 owns the row's selection state: the
// others send it their sample keys (step 1), receive the two thresholds
// (step 2), and send it their band keys and winner bits (step 3) through
// distributed shared memory; CTA 0 then selects within the band and emits
// (step 4).  Three cluster barriers in all.  If the band missed the k-th
// score, CTA 0 selects exactly over the whole row read back from memory.
__device__ __forceinline__ void st_dsmem_f32(uint32_t a, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void st_dsmem_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_add_dsmem_u32(uint32_t a, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(a), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void red_or_dsmem_u32(uint32_t a, uint32_t v) {
  asm volatile("red.shared::cluster.or.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

struct RowcShared {
  RowSel sh;
  float thr[2];        // t_hi, t_lo (sent by CTA 0)
  int band_ok;         // the sample gave thresholds
  uint32_t base;       // this CTA's first band slot in CTA 0
  uint32_t red_a[32], red_b[32];
};

// Emission of CTA 0: winners and the first krem ties of the masks, ascending.
template <int NT>
__device__ void emit_masks(RowSel &sh, const uint32_t *win, const uint32_t *tie, int nwords, int krem, int V, int k,
                           int32_t *out) {
  const int tid = threadIdx.x;
  const int wpt = (nwords + NT - 1) / NT;
  const int w0 = tid * wpt;
  int my_ties = 0;
  for (int u = 0; u < wpt; ++u)
    if (w0 + u < nwords) my_ties += __popc(tie[w0 + u]);
  int ties_before = block_exclusive_scan<NT>(my_ties, sh.warp_buf, &sh.scan_tot);
  int my_sel = 0;
  {
    int tb = ties_before;
    for (int u = 0; u < wpt; ++u)
      if (w0 + u < nwords) {
        const int nt = __popc(tie[w0 + u]);
        my_sel += __popc(win[w0 + u]) + max(0, min(nt, krem - tb));
        tb += nt;
      }
  }
  int at = block_exclusive_scan<NT>(my_sel, sh.warp_buf, &sh.scan_tot);
  for (int u = 0; u < wpt; ++u) {
    const int w = w0 + u;
    if (w >= nwords) break;
    uint32_t wm = win[w], tm = tie[w];
    while (wm | tm) {
      const int bw = wm ? __ffs(wm) - 1 : 32, bt = tm ? __ffs(tm) - 1 : 32;
      if (bw < bt) {
        out[at++] = w * 32 + bw;
        wm &= wm - 1u;
      } else {
        if (ties_before < krem) out[at++] = w * 32 + bt;
        ++ties_before;
        tm &= tm - 1u;
      }
    }
  }
  const int K = V < k ? V : k;
  for (int i = K + tid; i < k; i += NT) out[i] = -1;
}

// Grid: C CTAs per row, cluster (C,1,1).  Dynamic shared memory: 2 * words +
// 2 * kRowCand + C * NT words (masks, band, samples; used in CTA 0).
template <int NT>
__global__ void __launch_bounds__(NT) topk_rowc(TopkParams p) {
  constexpr int NW = NT / 32;
  extern __shared__ __align__(16) uint32_t dyn[];
  __shared__ RowcShared rs;
  RowSel &sh = rs.sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t C = cluster_nctarank(), rank = cluster_ctarank();
  const int row = blockIdx.x / C;
  const int V = p.fixed_len > 0 ? p.fixed_len : (p.start_pos + row % p.n_q + 1) / p.m;
  const int nwords = (V + 31) >> 5;
  const int per_cta = 32 * NT;
  const int base = (int)rank * per_cta;                  // first key of this CTA
  uint32_t *win = dyn;                                   // [words]        (CTA 0)
  uint32_t *tie = dyn + p.slice;                         // [words]        (CTA 0)
  uint32_t *band_key = dyn + 2 * p.slice;                // [kRowCand]     (CTA 0)
  uint32_t *band_idx = band_key + kRowCand;              // [kRowCand]     (CTA 0)
  float *samples = reinterpret_cast<float *>(band_idx + kRowCand);   // [C * NT] (CTA 0)
  int32_t *out = p.idx_out + (long long)row * p.out_stride;
  const unsigned long long st_entry = global_ns();
  pdl_wait();
  const unsigned long long st_ready = global_ns();
  // every row of a launch has V > k (the host sends short rows elsewhere)
  const float *src = p.scores + (long long)row * p.in_stride;
  float x[kRowRegs][4];
  const bool vec = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
#pragma unroll
  for (int j = 0; j < kRowRegs; ++j) {
    const int i = base + 4 * tid + 4 * NT * j;
    if (vec && i + 3 < V) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(src + i));
      x[j][0] = v.x; x[j][1] = v.y; x[j][2] = v.z; x[j][3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) x[j][e] = i + e < V ? __ldg(src + i + e) : 0.f;
    }
  }
  if (rank == 0) {
    for (int w = tid; w < nwords; w += NT) { win[w] = 0u; tie[w] = 0u; }
    for (int i = tid; i < kBinsMax; i += NT) sh.hist[i] = 0u;
    if (tid == 0) { sh.s_above = 0; sh.s_nc = 0; }
  }
  // ---- 1. one sample key per thread into CTA 0 (NaN marks "no key")
  {
    const int js = tid % kRowRegs;
    const int is = base + 4 * tid + 4 * NT * js;
    float sv = __uint_as_float(0x7FC00000u);
#pragma unroll
    for (int j = 0; j < kRowRegs; ++j)
      if (j == js && is < V) sv = x[j][0];
    st_dsmem_f32(cluster_map(smem_u32(samples + rank * NT + tid), 0), sv);
  }
  cluster_sync();
  // ---- 2. CTA 0: thresholds from the sample, sent to every CTA
  if (rank == 0) {
    const int S = (int)C * NT;
    uint32_t smin = 0xFFFFFFFFu, smax = 0u;
    int ns = 0;
    for (int i = tid; i < S; i += NT) {
      const float v = samples[i];
      if (v == v) {
        const uint32_t kk = order_bits(__float_as_uint(v));
        smin = min(smin, kk);
        smax = max(smax, kk);
        ++ns;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      smin = min(smin, __shfl_xor_sync(0xffffffffu, smin, o));
      smax = max(smax, __shfl_xor_sync(0xffffffffu, smax, o));
      ns += __shfl_xor_sync(0xffffffffu, ns, o);
    }
    if (lane == 0) { rs.red_a[warp] = smin; rs.red_b[warp] = smax; sh.warp_buf[warp] = ns; }
    __syncthreads();
    smin = rs.red_a[0]; smax = rs.red_b[0]; ns = sh.warp_buf[0];
    for (int w = 1; w < NW; ++w) { smin = min(smin, rs.red_a[w]); smax = max(smax, rs.red_b[w]); ns += sh.warp_buf[w]; }
    __syncthreads();
    const float lo = key_float(smin), hi = key_float(smax);
    const float scale = (float)kBinsMax / (hi - lo);
    const bool ok = ns >= 64 && smin != smax && scale > 0.f && scale < INFINITY;
    float t_hi = 0.f, t_lo = 0.f;
    if (ok) {
      for (int i = tid; i < S; i += NT) {
        const float v = samples[i];
        if (v == v) {
          const float f = (key_float(order_bits(__float_as_uint(v))) - lo) * scale;
          atomicAdd(&sh.hist[f >= (float)(kBinsMax - 1) ? (uint32_t)(kBinsMax - 1) : (f > 0.f ? (uint32_t)f : 0u)], 1u);
        }
      }
      __syncthreads();
      const float q = (float)p.k * (float)ns / (float)V;
      const int r_hi = max(1, (int)floorf(q - 3.f * sqrtf(q)));
      const int r_lo = min(ns, (int)ceilf(q + 3.f * sqrtf(q) + 2.f));
      row_find_digit<NT>(sh.hist, kBinsMax, r_hi, sh.warp_buf, &sh.scan_tot, sh.res);
      const int b_hi = sh.res[0];
      __syncthreads();
      row_find_digit<NT>(sh.hist, kBinsMax, r_lo, sh.warp_buf, &sh.scan_tot, sh.res);
      const int b_lo = sh.res[0];
      __syncthreads();
      for (int i = tid; i < kBinsMax; i += NT) sh.hist[i] = 0u;
      t_hi = lo + (float)(b_hi + 1) / scale;
      t_lo = lo + (float)b_lo / scale;
    }
    if (tid < (int)C) {
      const uint32_t r = (uint32_t)tid;
      st_dsmem_f32(cluster_map(smem_u32(&rs.thr[0]), r), t_hi);
      st_dsmem_f32(cluster_map(smem_u32(&rs.thr[1]), r), t_lo);
      st_dsmem_u32(cluster_map(smem_u32(&rs.band_ok), r), ok ? 1u : 0u);
    }
  }
  cluster_sync();
  // ---- 3. every CTA: winners' bits and band keys into CTA 0
  if (rs.band_ok) {
    const float t_hi = rs.thr[0], t_lo = rs.thr[1];
    int above = 0, inband = 0;
#pragma unroll
    for (int j = 0; j < kRowRegs; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool valid = base + 4 * tid + 4 * NT * j + e < V;
        const float v = x[j][e];
        above += (valid && v > t_hi) ? 1 : 0;
        inband += (valid && v <= t_hi && v >= t_lo) ? 1 : 0;
      }
    const int off = block_exclusive_scan<NT>(inband, sh.warp_buf, &sh.scan_tot);
    const int tot = sh.scan_tot;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
    if (lane == 0 && above) atom_add_dsmem_u32(cluster_map(smem_u32(&sh.s_above), 0), (uint32_t)above);
    if (tid == 0) rs.base = tot ? atom_add_dsmem_u32(cluster_map(smem_u32(&sh.s_nc), 0), (uint32_t)tot) : 0u;
    __syncthreads();
    int at = (int)rs.base + off;
    if (above | inband) {
      const uint32_t wmap = cluster_map(smem_u32(win), 0);
      const uint32_t kmap = cluster_map(smem_u32(band_key), 0);
      const uint32_t imap = cluster_map(smem_u32(band_idx), 0);
#pragma unroll
      for (int j = 0; j < kRowRegs; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = base + 4 * tid + 4 * NT * j + e;
          const float v = x[j][e];
          if (i < V && v > t_hi) {
            red_or_dsmem_u32(wmap + 4u * (uint32_t)(i >> 5), 1u << (i & 31));
          } else if (i < V && v >= t_lo) {
            if (at < kRowCand) {
              st_dsmem_u32(kmap + 4u * (uint32_t)at, order_bits(__float_as_uint(v)));
              st_dsmem_u32(imap + 4u * (uint32_t)at, (uint32_t)i);
            }
            ++at;
          }
        }
    }
  }
  cluster_sync();   // after this no CTA touches another's shared memory
  // the attention may now start its prologue: scheduling it earlier let its
  // CTAs take the SMs that clusters still waiting for placement needed
  pdl_trigger();
  if (rank == 0) {
    // ---- 4. CTA 0: exact selection within the band, or over the whole row
    const int na = sh.s_above, nc = sh.s_nc;
    const bool banded = rs.band_ok && na < p.k && na + nc >= p.k && nc <= kRowCand;
    int krem;
    uint32_t T;
    if (banded) {
      uint32_t cmin = 0xFFFFFFFFu, cmax = 0u;
      for (int i = tid; i < nc; i += NT) { cmin = min(cmin, band_key[i]); cmax = max(cmax, band_key[i]); }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        cmin = min(cmin, __shfl_xor_sync(0xffffffffu, cmin, o));
        cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
      }
      if (lane == 0) { rs.red_a[warp] = cmin; rs.red_b[warp] = cmax; }
      __syncthreads();
      cmin = rs.red_a[0]; cmax = rs.red_b[0];
      for (int w = 1; w < NW; ++w) { cmin = min(cmin, rs.red_a[w]); cmax = max(cmax, rs.red_b[w]); }
      krem = p.k - na;
      T = radix_select<NT>(sh, cmin, cmax, &krem, [&](auto f) {
        for (int i = tid; i < nc; i += NT) f(band_key[i]);
      });
      for (int i = tid; i < nc; i += NT) {
        const uint32_t kk = band_key[i], ix = band_idx[i];
        if (kk > T) atomicOr(&win[ix >> 5], 1u << (ix & 31));
        else if (kk == T) atomicOr(&tie[ix >> 5], 1u << (ix & 31));
      }
    } else {
      // the whole row, read back from memory (rare: heavy ties, a bad sample)
      for (int w = tid; w < nwords; w += NT) win[w] = 0u;
      uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
      for (int i = tid; i < V; i += NT) {
        const uint32_t kk = order_bits(__float_as_uint(src[i]));
        kmin = min(kmin, kk);
        kmax = max(kmax, kk);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      }
      if (lane == 0) { rs.red_a[warp] = kmin; rs.red_b[warp] = kmax; }
      __syncthreads();
      kmin = rs.red_a[0]; kmax = rs.red_b[0];
      for (int w = 1; w < NW; ++w) { kmin = min(kmin, rs.red_a[w]); kmax = max(kmax, rs.red_b[w]); }
      krem = p.k;
      T = radix_select<NT>(sh, kmin, kmax, &krem, [&](auto f) {
        for (int i = tid; i < V; i += NT) f(order_bits(__float_as_uint(src[i])));
      });
      for (int i = tid; i < V; i += NT) {
        const uint32_t kk = order_bits(__float_as_uint(src[i]));
        if (kk > T) atomicOr(&win[i >> 5], 1u << (i & 31));
        else if (kk == T) atomicOr(&tie[i >> 5], 1u << (i & 31));
      }
    }
    __syncthreads();
    emit_masks<NT>(sh, win, tie, nwords, krem, V, p.k, out);
  }
  if (step_trace_on()) {
    __syncthreads();
    if (tid == 0) step_trace_record(ST_TOPK, st_entry, st_ready);
  }
}

template <int NT>
int launch_topk_rowc_t(const TopkParams &t, long long rows, int Vmax, int C, cudaStream_t s) {
  const int words = (Vmax + 31) / 32;
  const size_t smem = (size_t)(2 * words + 2 * kRowCand + C * NT) * 4;
  static std::atomic<bool> attr_dev[kMaxDevices];
  std::atomic<bool> &attr = attr_dev[device_slot()];
  if (!attr) {
    const int max_words = kClusterMax * 32 * NT / 32;
    const cudaError_t e = cudaFuncSetAttribute(topk_rowc<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (2 * max_words + 2 * kRowCand + kClusterMax * NT) * 4);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "top-k cluster-row smem attribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  LaunchScope ls("topk", s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(rows * C), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  TopkParams tp = t;
  tp.slice = words;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_rowc<NT>, tp);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(HCA_ERR_CUDA, "topk_rowc launch: %s", cudaGetErrorString(e));
  }
  return ls.done();
}
// Rows all longer than k and few of them (decode): a cluster of C CTAs per
// row, C the smallest power of two (<= 8) giving every CTA at most 32 * NT
// keys.  HCA_ERR_UNSUPPORTED when the rows do not fit.
int launch_topk_rowc(const TopkParams &t, long long rows, int Vmax, cudaStream_t s) {
  const int NTs[2] = {128, 1024};
  for (int v = 0; v < 2; ++v) {
    const int NT = NTs[v];
    int C = 1;
    while (C < kClusterMax && (long long)C * 32 * NT < Vmax) C *= 2;
    if ((long long)C * 32 * NT < Vmax) continue;
    if (C < 2) C = 2;
    return NT == 128 ? launch_topk_rowc_t<128>(t, rows, Vmax, C, s) : launch_topk_rowc_t<1024>(t, rows, Vmax, C, s);
  }
  return HCA_ERR_UNSUPPORTED;
}

template <int NT, int RR>
int launch_topk_row_t(const TopkParams &t, long long rows, int Vmax, cudaStream_t s) {
  const int words = (Vmax + 31) / 32;
  const size_t smem = (size_t)(2 * words + 2 * kRowCand) * 4;
  static std::atomic<bool> attr_dev[kMaxDevices];
  std::atomic<bool> &attr = attr_dev[device_slot()];
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(topk_row<NT, RR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (2 * (kRowMax / 32) + 2 * kRowCand) * 4);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "top-k row smem attribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  LaunchScope ls("topk", s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)rows, 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  TopkParams tp = t;
  tp.slice = words;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_row<NT, RR>, tp);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(HCA_ERR_CUDA, "topk_row launch: %s", cudaGetErrorString(e));
  }
  return ls.done();
}
// A warp per row for many rows of up to kRowMax keys (HCA_ERR_UNSUPPORTED otherwise).
int launch_topk_warp(const TopkParams &t, long long rows, int Vmax, cudaStream_t s) {
  if (Vmax > kRowMax || rows > 0x7FFFFFFFLL) return HCA_ERR_UNSUPPORTED;
  const size_t smem = kWarpRowWarps * sizeof(WarpRowSmem);
  static std::atomic<bool> attr_dev[kMaxDevices];
  std::atomic<bool> &attr = attr_dev[device_slot()];
  if (!attr) {
    // two CTAs per SM: the whole unified L1 / shared array as shared memory
    cudaError_t e = cudaFuncSetAttribute(topk_warp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(topk_warp, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "top-k warp smem attribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  LaunchScope ls("topk", s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)((rows + kWarpRowWarps - 1) / kWarpRowWarps), 1, 1);
  cfg.blockDim = dim3(kWarpRowWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_warp, t);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(HCA_ERR_CUDA, "topk_warp launch: %s", cudaGetErrorString(e));
  }
  return ls.done();
}
// One CTA per row for rows of up to kRowMax keys (HCA_ERR_UNSUPPORTED otherwise);
// the longest rows take 64 keys per thread in 512 threads (no register spills).
int launch_topk_row(const TopkParams &t, long long rows, int Vmax, cudaStream_t s) {
  if (Vmax > kRowMax || rows > 0x7FFFFFFFLL) return HCA_ERR_UNSUPPORTED;
  if (Vmax <= 32 * 128) return launch_topk_row_t<128, 8>(t, rows, Vmax, s);
  if (Vmax <= 32 * 256) return launch_topk_row_t<256, 8>(t, rows, Vmax, s);
  if (Vmax <= 32 * 512) return launch_topk_row_t<512, 8>(t, rows, Vmax, s);
  return launch_topk_row_t<512, 16>(t, rows, Vmax, s);
}

struct TopkPlan {
  int C, n_seg, seg_len, slice;
};
// Cluster size, segments and per-CTA slice for rows of up to Vmax keys: grow
// the cluster (keeping >= 1024 keys per CTA) until the grid covers the SMs
// twice or the row fits one segment of C * kSliceMax keys.
TopkPlan plan_topk(long long rows, long long Vmax) {
  TopkPlan t{};
  int C = 1;
  const long long want = 2LL * num_sms();
  while (C < kClusterMax && Vmax >= 2048LL * C && (rows * C < want || (long long)C * kSliceMax < Vmax)) C *= 2;
  t.C = C;
  const long long per_seg = (long long)C * kSliceMax;
  t.n_seg = (int)max(1LL, (Vmax + per_seg - 1) / per_seg);
  long long seg_len = (Vmax + t.n_seg - 1) / t.n_seg;
  seg_len = ((seg_len + 4LL * C - 1) / (4LL * C)) * (4LL * C);
  t.seg_len = (int)max(seg_len, 4LL * C);
  t.slice = t.seg_len / C;
  return t;
}
size_t topk_smem(const TopkPlan &t) { return (size_t)(t.slice + kCandMax) * 4; }
int ensure_topk_smem() {
  static std::atomic<bool> done_dev[kMaxDevices];
  std::atomic<bool> &done = done_dev[device_slot()];
  if (!done) {
    const cudaError_t e = cudaFuncSetAttribute(topk_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (kSliceMax + kCandMax) * 4);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "top-k smem attribute: %s", cudaGetErrorString(e));
    done = true;
  }
  return HCA_OK;
}
int launch_topk_cluster(const char *name, const TopkParams &t, const TopkPlan &pl, long long rows, cudaStream_t s) {
  LaunchScope ls(name, s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(rows * pl.n_seg * pl.C), 1, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = topk_smem(pl);
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = pl.C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_cluster, t);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(HCA_ERR_CUDA, "%s launch: %s", name, cudaGetErrorString(e));
  }
  return ls.done();
}

}  // namespace

int launch_index_scores(const IndexParams &p, cudaStream_t s) {
  const int Vmax = (p.start_pos + p.n_q) / p.m;
  if (Vmax == 0) return HCA_OK;
  dim3 grid((Vmax + kScoreThreads - 1) / kScoreThreads, (p.n_q + kQB - 1) / kQB, p.B);
  const size_t smem = (size_t)(kQB * p.n_hI * p.c_I + kQB * p.n_hI) * sizeof(float);
  LaunchScope ls_("index_scores_simt", s);
  if (p.q_dtype == HCA_F32) {
    if (p.key_dtype == HCA_F32) index_scores_simt<float, float><<<grid, kScoreThreads, smem, s>>>(p);
    else index_scores_simt<float, __nv_bfloat16><<<grid, kScoreThreads, smem, s>>>(p);
  } else {
    if (p.key_dtype == HCA_F32) index_scores_simt<__nv_bfloat16, float><<<grid, kScoreThreads, smem, s>>>(p);
    else index_scores_simt<__nv_bfloat16, __nv_bfloat16><<<grid, kScoreThreads, smem, s>>>(p);
  }
  return ls_.done();
}


// FP4 path: the rotated, quantised q^I (bf16) after everything else.
size_t fp4_q_bytes(const IndexParams &p) {
  return p.key_dtype == HCA_FP4 ? (((size_t)p.B * p.n_q * p.n_hI * 64 * 2 + 255) & ~(size_t)255) : 0;
}

size_t topk_workspace_bytes(const IndexParams &p) {
  const long long rows = (long long)p.B * p.n_q;
  const long long Vmax = (p.start_pos + p.n_q) / p.m;
  const TopkPlan pl = plan_topk(rows, Vmax);
  size_t b = (size_t)rows * (size_t)Vmax * sizeof(float);           // scores
  b = (b + 255) & ~(size_t)255;
  if (pl.n_seg > 1 && !(Vmax <= kRowMax && g_topk_kernel != 3)) {
    const size_t c = (size_t)rows * pl.n_seg * p.k;
    b += 2 * ((c * sizeof(int32_t) + 255) & ~(size_t)255);          // winners' indices and keys
  }
  return b + fp4_q_bytes(p);
}

int run_index_topk(const IndexParams &ip, int32_t *idx, float *user_scores, long long user_stride,
                   void *ws, size_t ws_bytes, cudaStream_t s) {
  if (ws_bytes < topk_workspace_bytes(ip)) return fail(HCA_ERR_INVALID, "workspace too small");
  const long long rows = (long long)ip.B * ip.n_q;
  const int Vmax = (ip.start_pos + ip.n_q) / ip.m;
  IndexParams p = ip;
  char *w = static_cast<char *>(ws);
  if (user_scores) {
    p.scores = user_scores;
    p.score_stride = user_stride;
  } else {
    p.scores = reinterpret_cast<float *>(w);
    p.score_stride = Vmax;
  }
  size_t off = ((size_t)rows * (size_t)Vmax * sizeof(float) + 255) & ~(size_t)255;
  int rc = ensure_topk_smem();
  if (rc) return rc;
  if (ip.key_dtype == HCA_FP4) {
    // FP4 path: rotate and quantise q^I into the end of the workspace, then
    // score the exact bf16 images of both FP4 operands and round to bf16
    const size_t qb = fp4_q_bytes(ip);
    __nv_bfloat16 *q4 = reinterpret_cast<__nv_bfloat16 *>(w + topk_workspace_bytes(ip) - qb);
    rc = launch_fp4_rotate_quant(ip.qI, ip.q_dtype, (long long)ip.B * ip.n_q * ip.n_hI, q4, s);
    if (rc) return rc;
    p.qI = q4;
    p.q_dtype = HCA_BF16;
    p.key_dtype = HCA_BF16;
    p.round_bf16 = 1;
  }
  rc = launch_index_scores_tc(p, s);
  if (rc == HCA_ERR_UNSUPPORTED) rc = launch_index_scores(p, s);
  if (rc) return rc;
  const TopkPlan pl = plan_topk(rows, Vmax);
  TopkParams t{};
  t.rows = (int)rows; t.k = ip.k; t.scores = p.scores; t.in_stride = p.score_stride;
  t.n_q = ip.n_q; t.start_pos = ip.start_pos; t.m = ip.m;
  t.n_seg = pl.n_seg; t.seg_len = pl.seg_len; t.slice = pl.slice;
  const int force = g_topk_kernel;
  // few rows, all longer than k (decode): a cluster per row
  const int Vmin = (ip.start_pos + 1) / ip.m;
  if ((force == 0 && Vmin > ip.k && rows * 8 <= 2LL * num_sms() && Vmax > kRowMax) || (force == 4 && Vmin > ip.k)) {
    t.idx_out = idx; t.out_stride = ip.k;
    rc = launch_topk_rowc(t, rows, Vmax, s);
    if (rc != HCA_ERR_UNSUPPORTED) return rc;
  }
  // many rows (prefill): a warp per row
  if (((force == 0 && rows >= 2LL * num_sms()) || force == 2) && Vmax <= kRowMax) {
    t.idx_out = idx; t.out_stride = ip.k;
    return launch_topk_warp(t, rows, Vmax, s);
  }
  if ((force == 0 || force == 1) && Vmax <= kRowMax) {
    t.idx_out = idx; t.out_stride = ip.k;
    return launch_topk_row(t, rows, Vmax, s);
  }
  if (pl.n_seg == 1) {
    t.idx_out = idx; t.out_stride = ip.k;
    return launch_topk_cluster("topk", t, pl, rows, s);
  }
  // pass 1: the winners of every segment, with their order keys
  const int clen = pl.n_seg * ip.k;
  const size_t c = (size_t)rows * clen;
  int32_t *cidx = reinterpret_cast<int32_t *>(w + off);
  off += (c * sizeof(int32_t) + 255) & ~(size_t)255;
  uint32_t *ckey = reinterpret_cast<uint32_t *>(w + off);
  t.idx_out = cidx; t.key_out = ckey; t.out_stride = clen;
  rc = launch_topk_cluster("topk_pass1", t, pl, rows, s);
  if (rc) return rc;
  // pass 2: merge the segments' winners (segment order is index order)
  const TopkPlan pl2 = plan_topk(rows, clen);
  if (pl2.n_seg != 1) return fail(HCA_ERR_UNSUPPORTED, "top-k candidate list too long (%d)", clen);
  TopkParams t2{};
  t2.rows = (int)rows; t2.k = ip.k; t2.keys = ckey; t2.cand_idx = cidx; t2.in_stride = clen;
  t2.fixed_len = clen; t2.n_q = 1; t2.m = 1;
  t2.n_seg = 1; t2.seg_len = pl2.seg_len; t2.slice = pl2.slice;
  t2.idx_out = idx; t2.out_stride = ip.k;
  return launch_topk_cluster("topk_pass2", t2, pl2, rows, s);
}


// ------------------------------------------------- static-scratch variant
// Scratch for callers that cannot hand in a workspace: code that runs while
// the caller's device allocator is itself busy (an out-of-memory handler, an
// allocator hook), hosts whose device memory is reserved up front with no
// room for a per-call buffer, and loops that must not call cudaMalloc /
// cudaFree because those calls synchronise the device.  One array per device
// (per process): calls that overlap in time on one device -- two streams, two
// host threads, or a graph replay next to a direct call -- would share it and
// race, so such callers must order their calls (one stream, or events).
// Nothing in it must start at zero: the scorer writes every visible score of
// every row before the selection reads it, and a segmented selection's first
// launch writes every winner slot (padding included) before the merge reads it.
namespace {
static __device__ __align__(256) unsigned char g_index_topk_scratch[HCA_STATIC_SCRATCH_BYTES];

// Device address of the scratch on the current device, looked up once per
// device (the lookup may load the module, so it must not run during capture).
int static_scratch(void **out) {
  static std::mutex mu;
  static void *cached[64] = {nullptr};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(HCA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress((void **)&ptr, g_index_topk_scratch);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    cached[dev] = ptr;
  }
  *out = cached[dev];
  return HCA_OK;
}
}  // namespace

int run_index_topk_static(const IndexParams &p, int32_t *idx, float *user_scores, long long user_stride,
                          cudaStream_t s) {
  const size_t need = topk_workspace_bytes(p);
  if (need > (size_t)HCA_STATIC_SCRATCH_BYTES)
    return fail(HCA_ERR_INVALID,
                "csa_index_topk_static_scratch: this call needs %zu bytes of scratch (B*n_q rows x %d visible "
                "entries x 4 bytes, plus segment winners), the static scratch holds %zu; use csa_index_topk",
                need, (p.start_pos + p.n_q) / p.m, (size_t)HCA_STATIC_SCRATCH_BYTES);
  void *scratch = nullptr;
  const int rc = static_scratch(&scratch);
  if (rc) return rc;
  return run_index_topk(p, idx, user_scores, user_stride, scratch, (size_t)HCA_STATIC_SCRATCH_BYTES, s);
}

int step_trace_set_index_topk(void *buf, unsigned long long cap) { return step_trace_set_here(buf, cap); }

}  // namespace hca

extern "C" int hca_topk_kernel(int mode) {
  using namespace hca;
  if (mode > 4) return fail(HCA_ERR_INVALID, "top-k kernel mode %d (0..4)", mode);
  const int prev = g_topk_kernel;
  if (mode >= 0) g_topk_kernel = mode;
  return prev;
}
