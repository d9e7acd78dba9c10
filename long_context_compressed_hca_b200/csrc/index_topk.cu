// index_topk.cu -- lightning-indexer scores and per-query top-k selection.
//
// Score (juejin "DeepSeek-V4 技术报告简要解读" §2.3.1(b), Eq.(16); 1zeryu
// "DeepSeek-V4：算法架构", Indexer):  I[t,s] = sum_h w[t,h] ReLU(q^I[t,h].K^I[s])
// for the entries visible to t ((s+1)*m <= t+1).
// Selection (Eq.(17)): the min(k, V_t) highest scores, ties broken towards the
// lower entry index, emitted in ascending index order and padded with -1.
//
// The selection is an exact radix select on the order-preserving uint32 image
// of the fp32 scores (4 passes of 8 bits over a row held in shared memory),
// followed by a stable compaction; rows longer than one block's shared memory
// are cut into chunks whose local winners are merged by a second pass.
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
    if (s < (t + 1) / p.m)
      p.scores[((long long)b * p.n_q + q0 + j) * p.score_stride + s] = acc[j] * kscale;
  }
}

// ------------------------------------------------------------------ top-k
constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;                 // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // >= 1 for every non-NaN float
}

// Exclusive scan of one int per thread over the block; returns the prefix and
// writes the block total to *total.
__device__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < kTopkWarps ? warp_tot[lane] : 0;
    int u = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, u, o);
      if (lane >= o) u += y;
    }
    if (lane < kTopkWarps) warp_tot[lane] = u - t;   // exclusive warp offsets
    if (lane == kTopkWarps - 1) *total = u;
  }
  __syncthreads();
  const int r = warp_tot[warp] + x - v;
  __syncthreads();
  return r;
}

// One block selects the top-k of one (row, chunk).  Elements are read from
// scores[row*stride + begin + i] for i < len; with cand_idx the element's
// index is cand_idx[same offset] (-1 = absent), else elem_offset + begin + i.
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkParams p, int chunk, int n_chunks,
                                                             long long out_chunk_stride) {
  extern __shared__ uint32_t keys[];        // [chunk]
  __shared__ uint32_t hist[kTopkWarps][256];
  __shared__ uint32_t total[256];
  __shared__ int warp_tot[32];
  __shared__ int s_total;
  __shared__ uint32_t s_digit;
  __shared__ int s_krem;

  const int row = blockIdx.x, ch = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int V;
  if (p.row_len) V = p.row_len[row];
  else V = (p.start_pos + row % p.n_q + 1) / p.m;
  const long long begin = (long long)ch * chunk;
  const int len = (int)max(0LL, min((long long)chunk, (long long)V - begin));
  const float *src = p.scores + (long long)row * p.score_stride + begin;
  const int32_t *csrc = p.cand_idx ? p.cand_idx + (long long)row * p.score_stride + begin : nullptr;

  int nvalid = 0;
  for (int i = tid; i < len; i += kTopkThreads) {
    const bool ok = csrc ? csrc[i] >= 0 : true;
    keys[i] = ok ? order_key(src[i]) : 0u;
    nvalid += ok;
  }
  block_exclusive_scan(nvalid, warp_tot, &s_total);
  nvalid = s_total;
  const int K = min(p.k, nvalid);

  uint32_t T = 0;      // threshold key
  int krem = 0;        // how many keys equal to T to keep (in list order)
  if (K > 0 && K < nvalid) {
    uint32_t prefix = 0, mask = 0;
    krem = K;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < kTopkWarps * 256; i += kTopkThreads) (&hist[0][0])[i] = 0;
      __syncthreads();
      const int trips = (len + kTopkThreads - 1) / kTopkThreads;
      for (int tr = 0; tr < trips; ++tr) {
        const int i = tr * kTopkThreads + tid;
        uint32_t bin = 256;
        if (i < len) {
          const uint32_t kk = keys[i];
          if (kk != 0 && (kk & mask) == prefix) bin = (kk >> shift) & 255u;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin != 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[warp][bin], __popc(peers));
      }
      __syncthreads();
      if (tid < 256) {
        uint32_t t = 0;
#pragma unroll
        for (int w = 0; w < kTopkWarps; ++w) t += hist[w][tid];
        total[tid] = t;
      }
      __syncthreads();
      if (warp == 0) {
        // lane l covers bins 255-8l .. 248-8l (descending); suffix sums from the top
        uint32_t loc[8], run = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { run += total[255 - 8 * lane - j]; loc[j] = run; }
        uint32_t incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t before = incl - run;   // keys in higher bins than this lane's
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t above = before + (j ? loc[j - 1] : 0u);   // strictly higher bins
          const uint32_t upto = before + loc[j];
          if (above < (uint32_t)krem && upto >= (uint32_t)krem) {
            s_digit = 255 - 8 * lane - j;
            s_krem = krem - (int)above;
          }
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= 255u << shift;
      krem = s_krem;
      __syncthreads();
    }
    T = prefix;
  }
  // stable compaction: keep key > T, and the first krem keys == T
  const int seg = (len + kTopkThreads - 1) / kTopkThreads;
  const int lo = min(len, tid * seg), hi = min(len, lo + seg);
  int ceq = 0;
  for (int i = lo; i < hi; ++i) ceq += (keys[i] == T && T != 0);
  const int eq_base = block_exclusive_scan(ceq, warp_tot, &s_total);
  int csel = 0, e = eq_base;
  for (int i = lo; i < hi; ++i) {
    const uint32_t kk = keys[i];
    if (kk == 0) continue;
    if (kk > T) ++csel;
    else if (kk == T && T != 0) { if (e < krem) ++csel; ++e; }
  }
  const int out_base = block_exclusive_scan(csel, warp_tot, &s_total);
  int32_t *out = p.idx_out + (long long)row * p.idx_stride + (long long)ch * out_chunk_stride;
  float *sout = p.score_out ? p.score_out + (long long)row * p.idx_stride + (long long)ch * out_chunk_stride
                            : nullptr;
  int o = out_base;
  e = eq_base;
  for (int i = lo; i < hi; ++i) {
    const uint32_t kk = keys[i];
    if (kk == 0) continue;
    bool take = kk > T;
    if (kk == T && T != 0) { take = e < krem; ++e; }
    if (take) {
      out[o] = csrc ? csrc[i] : (int32_t)(p.elem_offset + begin + i);
      if (sout) sout[o] = src[i];
      ++o;
    }
  }
  for (int i = K + tid; i < p.k; i += kTopkThreads) {
    out[i] = -1;
    if (sout) sout[i] = -INFINITY;
  }
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

namespace {
constexpr int kMaxChunk = 16384;     // 64 KB of keys per block in pass 1
constexpr int kMaxMerge = 32768;     // candidates per row in pass 2 (128 KB)
int topk_chunk_for(int rows, int Vmax, int k) {
  if (Vmax <= 0) return 1;
  int chunk = kMaxChunk;
  // with few rows, cut each row into more chunks so that every SM has work,
  // keeping each chunk >= 4k so the merge pass still reduces
  const int want_blocks = 2 * num_sms();
  while (chunk / 2 >= 4 * k && chunk / 2 >= 1024 &&
         (long long)rows * ((Vmax + chunk - 1) / chunk) < want_blocks &&
         (long long)((Vmax + chunk / 2 - 1) / (chunk / 2)) * k <= kMaxMerge)
    chunk /= 2;
  return chunk;
}
int ensure_topk_smem() {
  static bool done = false;
  if (!done) {
    const cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               kMaxMerge * 4);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "top-k smem attribute: %s", cudaGetErrorString(e));
    done = true;
  }
  return HCA_OK;
}
}  // namespace

size_t topk_workspace_bytes(const IndexParams &p) {
  const int rows = p.B * p.n_q;
  const int Vmax = (p.start_pos + p.n_q) / p.m;
  const int chunk = topk_chunk_for(rows, Vmax, p.k);
  const int n_chunks = (Vmax + chunk - 1) / chunk;
  size_t b = (size_t)rows * (size_t)Vmax * sizeof(float);           // scores
  b = (b + 255) & ~(size_t)255;
  if (n_chunks > 1) {
    size_t c = (size_t)rows * n_chunks * p.k;
    b += ((c * sizeof(int32_t) + 255) & ~(size_t)255) + ((c * sizeof(float) + 255) & ~(size_t)255);
  }
  return b;
}

int launch_topk(const TopkParams &p, cudaStream_t s) {
  (void)p; (void)s;
  return HCA_ERR_UNSUPPORTED;
}

int run_index_topk(const IndexParams &ip, int32_t *idx, float *user_scores, long long user_stride,
                   void *ws, size_t ws_bytes, cudaStream_t s) {
  if (ws_bytes < topk_workspace_bytes(ip)) return fail(HCA_ERR_INVALID, "workspace too small");
  const int rows = ip.B * ip.n_q;
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
  rc = launch_index_scores_tc(p, s);
  if (rc == HCA_ERR_UNSUPPORTED) rc = launch_index_scores(p, s);
  if (rc) return rc;
  const int chunk = topk_chunk_for(rows, Vmax, ip.k);
  const int n_chunks = Vmax > 0 ? (Vmax + chunk - 1) / chunk : 1;
  TopkParams t{};
  t.rows = rows; t.k = ip.k; t.scores = p.scores; t.score_stride = p.score_stride;
  t.n_q = ip.n_q; t.start_pos = ip.start_pos; t.m = ip.m;
  if (n_chunks <= 1) {
    t.idx_out = idx; t.idx_stride = ip.k;
    return HCA_LAUNCH("topk", s, topk_kernel<<<dim3(rows, 1), kTopkThreads, (size_t)max(chunk, 1) * 4, s>>>(t, chunk, 1, 0));
  }
  // pass 1: local winners of each chunk
  const size_t c = (size_t)rows * n_chunks * ip.k;
  int32_t *cidx = reinterpret_cast<int32_t *>(w + off);
  off += (c * sizeof(int32_t) + 255) & ~(size_t)255;
  float *cscore = reinterpret_cast<float *>(w + off);
  t.idx_out = cidx; t.score_out = cscore; t.idx_stride = (long long)n_chunks * ip.k;
  rc = HCA_LAUNCH("topk_pass1", s, topk_kernel<<<dim3(rows, n_chunks), kTopkThreads, (size_t)chunk * 4, s>>>(t, chunk, n_chunks, ip.k));
  if (rc) return rc;
  // pass 2: merge the candidate lists (chunk order == index order)
  const int clen = n_chunks * ip.k;
  if (clen > kMaxMerge) return fail(HCA_ERR_UNSUPPORTED, "top-k candidate list too long (%d)", clen);
  TopkParams t2{};
  t2.rows = rows; t2.k = ip.k; t2.scores = cscore; t2.score_stride = clen; t2.cand_idx = cidx;
  t2.row_len = nullptr; t2.n_q = 1; t2.start_pos = clen - 1; t2.m = 1;   // every row has clen elements
  t2.idx_out = idx; t2.idx_stride = ip.k;
  const size_t smem = (size_t)clen * 4;
  return HCA_LAUNCH("topk_pass2", s, topk_kernel<<<dim3(rows, 1), kTopkThreads, smem, s>>>(t2, clen, 1, 0));
}

}  // namespace hca
