// layer.cu -- one attention layer end to end: prefill from hidden states and
// single-token decode over the caller's cache.
//
// Prefill (juejin "DeepSeek-V4 技术报告简要解读" §2.3.1-§2.3.3; 1zeryu
// "DeepSeek-V4：算法架构", Q/K/V 映射, Compressor, Indexer, Sparse Attention):
//   C/Z = H W_comp^T (fp32)            -> compressed entries (norm, RoPE at i*m)
//   indexer C/Z = H W_compI^T (CSA)    -> indexer keys
//   c^Q = RMSNorm(H W_DQ^T); q = per-head RMS(c^Q W_UQ^T), RoPE at t
//   q^I = c^Q W_IUQ^T, RoPE at t; w^I = H W_w^T * c_I^-1/2 n_hI^-1/2   (CSA)
//   window kv = RMSNorm(H W_KV^T), RoPE at t
//   CSA: scores + top-k; attend over window + selected / all visible entries.
// Decode (Compressor / Indexer decode branches): the token's projected rows
// are appended to the window ring and the compressor states; an entry is
// emitted when its block completes; then score, select and attend.
#include "common.cuh"
#include "internal.h"

namespace hca {
namespace {

size_t esize(hca_dtype t) { return t == HCA_F32 ? 4 : ((t == HCA_BF16 || t == HCA_FP4) ? 2 : 1); }

struct Carver {
  char *base;
  size_t off = 0;
  explicit Carver(void *b) : base(static_cast<char *>(b)) {}
  void *take(size_t bytes) {
    void *p = base ? base + off : nullptr;
    off += (bytes + 255) & ~(size_t)255;
    return p;
  }
};

// Copy the last min(w, n) window rows of every sequence into the ring (slot p % w).
template <typename T>
__global__ void ring_fill_kernel(const T *kv, T *ring, int B, int n, int w, int c) {
  const int b = blockIdx.y;
  const int first = n > w ? n - w : 0;
  const int rows = n - first;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < (long long)rows * c;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / c), col = (int)(e % c);
    const int p = first + r;
    ring[((long long)b * w + p % w) * c + col] = kv[((long long)b * n + p) * c + col];
  }
}


struct Plan {
  // prefill buffers
  void *CZ, *CZI, *cQ32, *cQ, *q32, *q, *qI32, *qI, *wI, *kv32, *kvw, *kvc, *keyI, *keyI_scale, *idx, *topk_ws;
  size_t topk_bytes, total;
  int qchunk;
};

int plan_prefill(const hca_layer *L, int n, void *ws, Plan &P) {
  const hca_attn_desc &a = L->a;
  const bool csa = L->kind == HCA_LAYER_CSA, comp = L->kind != HCA_LAYER_SWA;
  const long long T = (long long)a.B * n;
  const int E = comp ? n / a.m : 0;
  const size_t es = esize(a.dtype);
  Carver cv(ws);
  P.CZ = comp ? cv.take(T * (csa ? 4 : 2) * a.c * 4) : nullptr;
  P.CZI = csa ? cv.take(T * 4 * a.c_I * 4) : nullptr;
  P.cQ32 = cv.take(T * L->d_c * 4);
  P.cQ = cv.take(T * L->d_c * es);
  P.qchunk = (int)(T < 8192 ? T : 8192);
  P.q32 = cv.take((size_t)P.qchunk * a.n_h * a.c * 4);
  P.q = cv.take(T * a.n_h * a.c * es);
  P.qI32 = csa ? cv.take(T * a.n_hI * a.c_I * 4) : nullptr;
  P.qI = csa ? cv.take(T * a.n_hI * a.c_I * es) : nullptr;
  P.wI = csa ? cv.take(T * a.n_hI * 4) : nullptr;
  P.kv32 = cv.take(T * a.c * 4);
  P.kvw = cv.take(T * a.c * es);
  P.kvc = comp ? cv.take((size_t)a.B * (E > 0 ? E : 1) * a.c * es) : nullptr;
  P.keyI = csa ? cv.take((size_t)a.B * (E > 0 ? E : 1) * a.c_I * es) : nullptr;
  P.keyI_scale = nullptr;
  P.idx = csa ? cv.take(T * a.k * 4) : nullptr;
  P.topk_bytes = 0;
  if (csa) {
    IndexParams ip{};
    ip.B = a.B; ip.n_q = n; ip.start_pos = 0; ip.m = a.m; ip.k = a.k; ip.n_hI = a.n_hI; ip.c_I = a.c_I;
    ip.key_dtype = a.idx_key_dtype;
    P.topk_bytes = topk_workspace_bytes(ip);
  }
  P.topk_ws = P.topk_bytes ? cv.take(P.topk_bytes) : nullptr;
  P.total = cv.off;
  return HCA_OK;
}

int check_layer(const hca_layer *L) {
  if (!L) return fail(HCA_ERR_INVALID, "null layer");
  const hca_attn_desc &a = L->a;
  if (a.B < 1 || a.n_h < 1 || a.c < 32 || a.c > 512 || a.c % 32 || a.rd % 8 || a.rd > a.c || a.w < 0 || a.m < 1)
    return fail(HCA_ERR_INVALID, "invalid attention shape");
  if (a.dtype != HCA_F32 && a.dtype != HCA_BF16) return fail(HCA_ERR_INVALID, "dtype must be f32 or bf16");
  if (L->kind == HCA_LAYER_CSA) {
    if (a.k < 1 || a.n_hI < 1 || a.c_I < 8 || a.c_I % 8 || a.rd_I % 8 || a.rd_I > a.c_I)
      return fail(HCA_ERR_INVALID, "invalid indexer shape");
    if (a.overlap != 1 && a.overlap != 0) return fail(HCA_ERR_INVALID, "overlap must be 0 or 1");
  }
  if (L->kind != HCA_LAYER_CSA && L->kind != HCA_LAYER_HCA && L->kind != HCA_LAYER_SWA)
    return fail(HCA_ERR_INVALID, "unknown layer kind");
  if (!L->sink) return fail(HCA_ERR_INVALID, "sink must be non-null");
  return HCA_OK;
}

float rope_theta(const hca_attn_desc &a) { return a.rope_theta > 0.f ? a.rope_theta : 10000.f; }
float eps_of(const hca_attn_desc &a) { return a.eps > 0.f ? a.eps : 1e-6f; }

}  // namespace
}  // namespace hca

using namespace hca;

extern "C" {

size_t hybrid_layer_forward_workspace_size(const hca_layer *L, int n) {
  if (check_layer(L) || n < 0) return 0;
  Plan P{};
  plan_prefill(L, n, nullptr, P);
  return P.total;
}

int hybrid_layer_forward(const hca_layer *L, const void *H, int n, hca_cache *cache, void *o, void *ws,
                         size_t ws_bytes, hca_stream_t stream) {
  int rc = check_layer(L);
  if (rc) return rc;
  const hca_attn_desc &a = L->a;
  const bool csa = L->kind == HCA_LAYER_CSA, comp = L->kind != HCA_LAYER_SWA;
  if (n < 0 || !H || !o) return fail(HCA_ERR_INVALID, "H and o must be non-null, n >= 0");
  if (L->d < 8 || L->d_c < 8) return fail(HCA_ERR_INVALID, "d and d_c must be >= 8");
  if (!L->W_DQ || !L->W_UQ || !L->W_KV || (comp && (!L->W_comp || !L->B_comp)) ||
      (csa && (!L->W_compI || !L->B_compI || !L->W_IUQ || !L->W_w)))
    return fail(HCA_ERR_INVALID, "missing layer weight");
  Plan P{};
  plan_prefill(L, n, nullptr, P);
  if (ws_bytes < P.total || !ws) return fail(HCA_ERR_INVALID, "workspace too small (%zu < %zu)", ws_bytes, P.total);
  plan_prefill(L, n, ws, P);
  if (n == 0) return HCA_OK;
  const int E = comp ? n / a.m : 0;
  if (cache && comp && cache->cap < E) return fail(HCA_ERR_INVALID, "cache cap < n/m");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long T = (long long)a.B * n;
  const hca_dtype dt = a.dtype;
  const size_t es = esize(dt);
  const float theta = rope_theta(a), eps = eps_of(a);

  // ---- compressed main KV
  void *kvc = P.kvc;
  int cap = E > 0 ? E : 1;
  // a mixed-precision cache is filled from the bf16 entries after compression
  if (cache && comp && !a.kv_mixed) { kvc = cache->kv_comp; cap = cache->cap; }
  if (comp) {
    const int ncz = csa ? 4 : 2;
    rc = launch_gemm(dt, H, L->d, L->W_comp, L->d, P.CZ, (long long)ncz * a.c, HCA_F32, (int)T, ncz * a.c, L->d, 1.f, s);
    if (rc) return rc;
    hca_compress_desc cd{};
    cd.B = a.B; cd.width = a.c; cd.m = a.m; cd.overlap = csa ? a.overlap : 0; cd.rd = a.rd;
    cd.flags = HCA_COMPRESS_NORM | HCA_COMPRESS_ROPE; cd.eps = eps; cd.rope_theta = theta;
    cd.in_dtype = HCA_F32; cd.out_dtype = dt;
    const float *CZ = static_cast<const float *>(P.CZ);
    const long long rs = (long long)ncz * a.c;
    const bool ov = cd.overlap != 0;
    // column blocks: CSA [Ca | Cb | Za | Zb]; HCA [C | Z]
    rc = csa_compress(&cd, 0, n, CZ, ov ? CZ + a.c : nullptr, CZ + (csa ? 2 : 1) * a.c,
                      ov ? CZ + 3 * a.c : nullptr, rs, rs * n, L->B_comp, ov ? L->B_comp + a.m * a.c : nullptr,
                      nullptr, kvc, nullptr, cap, cache ? cache->state_kv : nullptr,
                      cache ? cache->state_score : nullptr, stream);
    if (rc) return rc;
    if (cache && a.kv_mixed && E > 0) {
      rc = launch_kv_quant_mixed(P.kvc, dt, (long long)a.B * E, a.c, a.rd, cache->kv_comp, s, E, cache->cap);
      if (rc) return rc;
    }
  }
  // ---- indexer keys
  void *keyI = P.keyI;
  float *keyIs = nullptr;
  // without a cache the keys stay in the workspace in dtype, or FP4 (bf16 storage)
  hca_dtype kdt = a.idx_key_dtype == HCA_FP4 ? HCA_FP4 : dt;
  if (csa) {
    if (cache) { keyI = cache->key_I; keyIs = cache->key_I_scale; kdt = a.idx_key_dtype; }
    rc = launch_gemm(dt, H, L->d, L->W_compI, L->d, P.CZI, 4LL * a.c_I, HCA_F32, (int)T, 4 * a.c_I, L->d, 1.f, s);
    if (rc) return rc;
    hca_compress_desc cd{};
    cd.B = a.B; cd.width = a.c_I; cd.m = a.m; cd.overlap = a.overlap; cd.rd = a.rd_I;
    cd.flags = HCA_COMPRESS_NORM | HCA_COMPRESS_ROPE; cd.eps = eps; cd.rope_theta = theta;
    cd.in_dtype = HCA_F32; cd.out_dtype = kdt;
    const float *CZ = static_cast<const float *>(P.CZI);
    const long long rs = 4LL * a.c_I;
    const bool ov = a.overlap != 0;
    rc = csa_compress(&cd, 0, n, CZ, ov ? CZ + a.c_I : nullptr, CZ + 2 * a.c_I, ov ? CZ + 3 * a.c_I : nullptr, rs,
                      rs * n, L->B_compI, ov ? L->B_compI + a.m * a.c_I : nullptr, nullptr, keyI, keyIs, cap,
                      cache ? cache->stateI_kv : nullptr, cache ? cache->stateI_score : nullptr, stream);
    if (rc) return rc;
  }
  // ---- queries
  rc = launch_gemm(dt, H, L->d, L->W_DQ, L->d, P.cQ32, L->d_c, HCA_F32, (int)T, L->d_c, L->d, 1.f, s);
  if (rc) return rc;
  {
    RowOpParams r{};
    r.in = static_cast<const float *>(P.cQ32); r.in_stride = L->d_c; r.out = P.cQ; r.out_stride = L->d_c;
    r.out_dtype = dt; r.rows = (int)T; r.cols = L->d_c; r.norm = 1; r.eps = eps; r.rd = 0; r.theta = theta;
    r.rows_per_pos = 1; r.pos_mod = n; r.scale = 1.f;
    if ((rc = launch_row_op(r, s))) return rc;
  }
  const int HC = a.n_h * a.c;
  for (long long r0 = 0; r0 < T; r0 += P.qchunk) {
    const int rows = (int)((T - r0) < P.qchunk ? (T - r0) : P.qchunk);
    rc = launch_gemm(dt, static_cast<const char *>(P.cQ) + r0 * L->d_c * es, L->d_c, L->W_UQ, L->d_c, P.q32, HC,
                     HCA_F32, rows, HC, L->d_c, 1.f, s);
    if (rc) return rc;
    RowOpParams r{};
    r.in = static_cast<const float *>(P.q32); r.in_stride = a.c;
    r.out = static_cast<char *>(P.q) + r0 * HC * es; r.out_stride = a.c; r.out_dtype = dt;
    r.rows = rows * a.n_h; r.cols = a.c; r.norm = 1; r.eps = eps; r.rd = a.rd; r.theta = theta;
    r.pos0 = r0 % n; r.rows_per_pos = a.n_h; r.pos_mod = n; r.scale = 1.f;
    if ((rc = launch_row_op(r, s))) return rc;
  }
  if (csa) {
    const int HI = a.n_hI * a.c_I;
    rc = launch_gemm(dt, P.cQ, L->d_c, L->W_IUQ, L->d_c, P.qI32, HI, HCA_F32, (int)T, HI, L->d_c, 1.f, s);
    if (rc) return rc;
    RowOpParams r{};
    r.in = static_cast<const float *>(P.qI32); r.in_stride = a.c_I; r.out = P.qI; r.out_stride = a.c_I;
    r.out_dtype = dt; r.rows = (int)T * a.n_hI; r.cols = a.c_I; r.norm = 0; r.rd = a.rd_I; r.theta = theta;
    r.rows_per_pos = a.n_hI; r.pos_mod = n; r.scale = 1.f;
    if ((rc = launch_row_op(r, s))) return rc;
    const float wscale = 1.0f / sqrtf((float)a.c_I) / sqrtf((float)a.n_hI);
    rc = launch_gemm(dt, H, L->d, L->W_w, L->d, P.wI, a.n_hI, HCA_F32, (int)T, a.n_hI, L->d, wscale, s);
    if (rc) return rc;
  }
  // ---- window kv
  rc = launch_gemm(dt, H, L->d, L->W_KV, L->d, P.kv32, a.c, HCA_F32, (int)T, a.c, L->d, 1.f, s);
  if (rc) return rc;
  {
    RowOpParams r{};
    r.in = static_cast<const float *>(P.kv32); r.in_stride = a.c; r.out = P.kvw; r.out_stride = a.c;
    r.out_dtype = dt; r.rows = (int)T; r.cols = a.c; r.norm = 1; r.eps = eps; r.rd = a.rd; r.theta = theta;
    r.rows_per_pos = 1; r.pos_mod = n; r.scale = 1.f;
    if ((rc = launch_row_op(r, s))) return rc;
  }
  if (cache && a.w > 0 && cache->win && a.kv_mixed) {
    // the last min(w, n) window rows of every sequence as records in ring slot
    // p % w: at most two runs of consecutive slots per sequence
    const int rec = (int)kv_mixed_row_bytes(a.c, a.rd);
    const int first = n > a.w ? n - a.w : 0;
    for (int b = 0; b < a.B; ++b) {
      int p0 = first;
      while (p0 < n) {
        const int run = (a.w - p0 % a.w) < (n - p0) ? (a.w - p0 % a.w) : (n - p0);
        rc = launch_kv_quant_mixed(static_cast<const char *>(P.kvw) + ((long long)b * n + p0) * a.c * es, dt, run, a.c,
                                   a.rd, static_cast<char *>(cache->win) + ((long long)b * a.w + p0 % a.w) * rec, s);
        if (rc) return rc;
        p0 += run;
      }
    }
  } else if (cache && a.w > 0 && cache->win) {
    dim3 g(8, a.B);
    LaunchScope ls_("ring_fill", s);
    if (dt == HCA_F32) ring_fill_kernel<float><<<g, 256, 0, s>>>((const float *)P.kvw, (float *)cache->win, a.B, n, a.w, a.c);
    else ring_fill_kernel<__nv_bfloat16><<<g, 256, 0, s>>>((const __nv_bfloat16 *)P.kvw, (__nv_bfloat16 *)cache->win, a.B, n, a.w, a.c);
    if ((rc = ls_.done())) return rc;
  }
  // ---- select + attend (on the bf16 rows of this call, also with a mixed-precision cache)
  hca_attn_desc ad = a;
  ad.kv_mixed = 0;
  if (csa) {
    ad.idx_key_dtype = kdt;
    rc = csa_index_topk(&ad, P.qI, static_cast<const float *>(P.wI), keyI, keyIs, cap, n, 0,
                        static_cast<int32_t *>(P.idx), nullptr, 0, P.topk_ws, P.topk_bytes, stream);
    if (rc) return rc;
    return csa_attend(&ad, P.q, kvc, cap, static_cast<const int32_t *>(P.idx), P.kvw, 0, L->sink, n, 0, o,
                      nullptr, 0, stream);
  }
  if (comp)
    return hca_attend(&ad, P.q, kvc, cap, P.kvw, 0, L->sink, n, 0, o, nullptr, 0, stream);
  // pure sliding window: an HCA attend whose compressed set is empty
  ad.m = n + 1;
  return hca_attend(&ad, P.q, P.kvw, 1, P.kvw, 0, L->sink, n, 0, o, nullptr, 0, stream);
}

// ----------------------------------------------------------- context parallel
// A rank's share of a context-parallel prefill: tokens [t0, t0 + n_loc) of
// every sequence, with h = hybrid_cp_halo(L, t0) rows of the previous tokens.
namespace {
int cp_block_halo(const hca_layer *L) {
  return (L->kind == HCA_LAYER_CSA && L->a.overlap) ? L->a.m : 0;
}
int cp_check(const hca_layer *L, const void *H, int t0, int n_loc) {
  int rc = check_layer(L);
  if (rc) return rc;
  const hca_attn_desc &a = L->a;
  if (!H) return fail(HCA_ERR_INVALID, "H must be non-null");
  if (t0 < 0 || n_loc < 1) return fail(HCA_ERR_INVALID, "t0 must be >= 0 and n_loc >= 1");
  if (L->kind == HCA_LAYER_SWA) return fail(HCA_ERR_UNSUPPORTED, "context-parallel prefill needs a compressed layer");
  if (t0 % a.m) return fail(HCA_ERR_INVALID, "t0 (%d) must start a compression block (m = %d)", t0, a.m);
  if (cp_block_halo(L) > 0 && a.w - 1 < cp_block_halo(L))
    return fail(HCA_ERR_UNSUPPORTED, "the window (w = %d) must cover the overlap block (m = %d)", a.w, a.m);
  if (L->d < 8 || L->d_c < 8) return fail(HCA_ERR_INVALID, "d and d_c must be >= 8");
  return HCA_OK;
}
struct CpPlan {
  void *CZ, *CZI, *cQ32, *cQ, *q32, *q, *qI32, *qI, *wI, *kv32, *kvw, *idx, *topk_ws;
  size_t topk_bytes, total;
  int qchunk;
};
void plan_cp(const hca_layer *L, int t0, int n_loc, void *ws, CpPlan &P) {
  const hca_attn_desc &a = L->a;
  const bool csa = L->kind == HCA_LAYER_CSA;
  const int h = hybrid_cp_halo(L, t0);
  const long long R = (long long)a.B * (h + n_loc);   // rows with the halo
  const long long T = (long long)a.B * n_loc;         // the rank's own rows
  const size_t es = esize(a.dtype);
  Carver cv(ws);
  P.CZ = cv.take(R * (csa ? 4 : 2) * a.c * 4);
  P.CZI = csa ? cv.take(R * 4 * a.c_I * 4) : nullptr;
  P.cQ32 = cv.take(T * L->d_c * 4);
  P.cQ = cv.take(T * L->d_c * es);
  P.qchunk = (int)(n_loc < 8192 ? n_loc : 8192);
  P.q32 = cv.take((size_t)P.qchunk * a.n_h * a.c * 4);
  P.q = cv.take(T * a.n_h * a.c * es);
  P.qI32 = csa ? cv.take(T * a.n_hI * a.c_I * 4) : nullptr;
  P.qI = csa ? cv.take(T * a.n_hI * a.c_I * es) : nullptr;
  P.wI = csa ? cv.take(T * a.n_hI * 4) : nullptr;
  P.kv32 = cv.take(R * a.c * 4);
  P.kvw = cv.take(R * a.c * es);
  P.idx = csa ? cv.take(T * a.k * 4) : nullptr;
  P.topk_bytes = 0;
  if (csa) {
    IndexParams ip{};
    ip.B = a.B; ip.n_q = n_loc; ip.start_pos = t0; ip.m = a.m; ip.k = a.k; ip.n_hI = a.n_hI; ip.c_I = a.c_I;
    ip.key_dtype = a.idx_key_dtype;
    P.topk_bytes = topk_workspace_bytes(ip);
  }
  P.topk_ws = P.topk_bytes ? cv.take(P.topk_bytes) : nullptr;
  P.total = cv.off;
}
// Entries of the rank's complete blocks from the projected C/Z rows (with the
// halo): rows start at token t0 - h; the compression reads from t0 - hb (the
// previous block, whose b series the first entry needs) and writes entries
// t0/m .. (t0 + n_loc)/m - 1 to out slots 0 ...
int cp_compress_series(const hca_layer *L, int t0, int n_loc, int h, const float *CZ, int width, int ncz,
                       const float *Bias, hca_dtype out_dt, int rd, void *out, float *out_scale, long long out_cap,
                       cudaStream_t s) {
  const hca_attn_desc &a = L->a;
  const bool ov = L->kind == HCA_LAYER_CSA && a.overlap;
  const int hb = (ov && t0 > 0) ? a.m : 0;
  hca_compress_desc cd{};
  cd.B = a.B; cd.width = width; cd.m = a.m; cd.overlap = ov ? 1 : 0; cd.rd = rd;
  cd.flags = HCA_COMPRESS_NORM | HCA_COMPRESS_ROPE; cd.eps = eps_of(a); cd.rope_theta = rope_theta(a);
  cd.in_dtype = HCA_F32; cd.out_dtype = out_dt;
  const long long rs = (long long)ncz * width;
  const float *base = CZ + (long long)(h - hb) * rs;
  // column blocks: CSA [Ca | Cb | Za | Zb]; HCA [C | Z]
  const float *Ca = base, *Cb = ov ? base + width : nullptr;
  const float *Za = base + (ov ? 2 : 1) * width, *Zb = ov ? base + 3 * width : nullptr;
  CompressParams p{};
  int rc = compress_params(&cd, 0, hb + n_loc, Ca, Cb, Za, Zb, rs, rs * (h + n_loc), Bias,
                           ov ? Bias + a.m * width : nullptr, nullptr, out, out_scale, out_cap, nullptr, nullptr, &p);
  if (rc) return rc;
  p.e_first = hb / a.m;
  p.e_pos0 = (t0 - hb) / a.m;
  return launch_compress_prefill(p, s);
}
}  // namespace

int hybrid_cp_halo(const hca_layer *L, int t0) {
  if (!L || t0 <= 0) return 0;
  const int need = L->a.w - 1 > cp_block_halo(L) ? L->a.w - 1 : cp_block_halo(L);
  return need < t0 ? need : t0;
}

size_t hybrid_cp_workspace_size(const hca_layer *L, int t0, int n_loc) {
  if (check_layer(L) || t0 < 0 || n_loc < 1) return 0;
  CpPlan P{};
  plan_cp(L, t0, n_loc, nullptr, P);
  return P.total;
}

int hybrid_cp_compress(const hca_layer *L, const void *H, int t0, int n_loc, void *kv_comp, void *key_I,
                       float *key_I_scale, int out_cap, void *ws, size_t ws_bytes, hca_stream_t stream) {
  int rc = cp_check(L, H, t0, n_loc);
  if (rc) return rc;
  const hca_attn_desc &a = L->a;
  const bool csa = L->kind == HCA_LAYER_CSA;
  const int E_loc = n_loc / a.m;
  if (!L->W_comp || !L->B_comp || (csa && (!L->W_compI || !L->B_compI))) return fail(HCA_ERR_INVALID, "missing layer weight");
  if (E_loc > 0 && (!kv_comp || (csa && !key_I))) return fail(HCA_ERR_INVALID, "kv_comp and key_I must be non-null");
  if (out_cap < E_loc) return fail(HCA_ERR_INVALID, "out_cap (%d) < entries of the range (%d)", out_cap, E_loc);
  if (csa && a.idx_key_dtype == HCA_FP8E4M3 && !key_I_scale) return fail(HCA_ERR_INVALID, "fp8 keys need key_I_scale");
  CpPlan P{};
  plan_cp(L, t0, n_loc, nullptr, P);
  if (!ws || ws_bytes < P.total) return fail(HCA_ERR_INVALID, "workspace too small (%zu < %zu)", ws_bytes, P.total);
  plan_cp(L, t0, n_loc, ws, P);
  if (E_loc == 0) return HCA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int h = hybrid_cp_halo(L, t0);
  const int R = a.B * (h + n_loc);
  const int ncz = csa ? 4 : 2;
  rc = launch_gemm(a.dtype, H, L->d, L->W_comp, L->d, P.CZ, (long long)ncz * a.c, HCA_F32, R, ncz * a.c, L->d, 1.f, s);
  if (rc) return rc;
  rc = cp_compress_series(L, t0, n_loc, h, static_cast<const float *>(P.CZ), a.c, ncz, L->B_comp, a.dtype, a.rd,
                          kv_comp, nullptr, out_cap, s);
  if (rc || !csa) return rc;
  rc = launch_gemm(a.dtype, H, L->d, L->W_compI, L->d, P.CZI, 4LL * a.c_I, HCA_F32, R, 4 * a.c_I, L->d, 1.f, s);
  if (rc) return rc;
  return cp_compress_series(L, t0, n_loc, h, static_cast<const float *>(P.CZI), a.c_I, 4, L->B_compI, a.idx_key_dtype,
                            a.rd_I, key_I, key_I_scale, out_cap, s);
}

int hybrid_cp_attend(const hca_layer *L, const void *H, int t0, int n_loc, const void *kv_comp, const void *key_I,
                     const float *key_I_scale, int cap, void *o, void *ws, size_t ws_bytes, hca_stream_t stream) {
  int rc = cp_check(L, H, t0, n_loc);
  if (rc) return rc;
  const hca_attn_desc &a = L->a;
  const bool csa = L->kind == HCA_LAYER_CSA;
  if (!o) return fail(HCA_ERR_INVALID, "o must be non-null");
  if (!L->W_DQ || !L->W_UQ || !L->W_KV || (csa && (!L->W_IUQ || !L->W_w))) return fail(HCA_ERR_INVALID, "missing layer weight");
  const int Vmax = (t0 + n_loc) / a.m;
  if (cap < Vmax) return fail(HCA_ERR_INVALID, "cap (%d) < entries visible to the range (%d)", cap, Vmax);
  if (Vmax > 0 && (!kv_comp || (csa && !key_I))) return fail(HCA_ERR_INVALID, "kv_comp and key_I must be non-null");
  CpPlan P{};
  plan_cp(L, t0, n_loc, nullptr, P);
  if (!ws || ws_bytes < P.total) return fail(HCA_ERR_INVALID, "workspace too small (%zu < %zu)", ws_bytes, P.total);
  plan_cp(L, t0, n_loc, ws, P);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const hca_dtype dt = a.dtype;
  const size_t es = esize(dt);
  const float theta = rope_theta(a), eps = eps_of(a);
  const int h = hybrid_cp_halo(L, t0);
  const char *Hb = static_cast<const char *>(H);
  const long long hrow = (long long)L->d * es;
  // ---- queries of the rank's own tokens (per sequence: its rows follow the halo)
  for (int b = 0; b < a.B; ++b) {
    rc = launch_gemm(dt, Hb + ((long long)b * (h + n_loc) + h) * hrow, L->d, L->W_DQ, L->d,
                     static_cast<float *>(P.cQ32) + (long long)b * n_loc * L->d_c, L->d_c, HCA_F32, n_loc, L->d_c, L->d,
                     1.f, s);
    if (rc) return rc;
  }
  const long long T = (long long)a.B * n_loc;
  {
    RowOpParams r{};
    r.in = static_cast<const float *>(P.cQ32); r.in_stride = L->d_c; r.out = P.cQ; r.out_stride = L->d_c;
    r.out_dtype = dt; r.rows = (int)T; r.cols = L->d_c; r.norm = 1; r.eps = eps; r.rd = 0; r.theta = theta;
    r.rows_per_pos = 1; r.pos_mod = n_loc; r.scale = 1.f;
    if ((rc = launch_row_op(r, s))) return rc;
  }
  const int HC = a.n_h * a.c;
  for (long long r0 = 0; r0 < T; r0 += P.qchunk) {
    const int rows = (int)((T - r0) < P.qchunk ? (T - r0) : P.qchunk);
    rc = launch_gemm(dt, static_cast<const char *>(P.cQ) + r0 * L->d_c * es, L->d_c, L->W_UQ, L->d_c, P.q32, HC,
                     HCA_F32, rows, HC, L->d_c, 1.f, s);
    if (rc) return rc;
    RowOpParams r{};
    r.in = static_cast<const float *>(P.q32); r.in_stride = a.c;
    r.out = static_cast<char *>(P.q) + r0 * HC * es; r.out_stride = a.c; r.out_dtype = dt;
    r.rows = rows * a.n_h; r.cols = a.c; r.norm = 1; r.eps = eps; r.rd = a.rd; r.theta = theta;
    r.pos0 = r0 % n_loc; r.rows_per_pos = a.n_h; r.pos_mod = n_loc; r.pos_base = t0; r.scale = 1.f;
    if ((rc = launch_row_op(r, s))) return rc;
  }
  if (csa) {
    const int HI = a.n_hI * a.c_I;
    rc = launch_gemm(dt, P.cQ, L->d_c, L->W_IUQ, L->d_c, P.qI32, HI, HCA_F32, (int)T, HI, L->d_c, 1.f, s);
    if (rc) return rc;
    RowOpParams r{};
    r.in = static_cast<const float *>(P.qI32); r.in_stride = a.c_I; r.out = P.qI; r.out_stride = a.c_I;
    r.out_dtype = dt; r.rows = (int)T * a.n_hI; r.cols = a.c_I; r.norm = 0; r.rd = a.rd_I; r.theta = theta;
    r.rows_per_pos = a.n_hI; r.pos_mod = n_loc; r.pos_base = t0; r.scale = 1.f;
    if ((rc = launch_row_op(r, s))) return rc;
    const float wscale = 1.0f / sqrtf((float)a.c_I) / sqrtf((float)a.n_hI);
    for (int b = 0; b < a.B; ++b) {
      rc = launch_gemm(dt, Hb + ((long long)b * (h + n_loc) + h) * hrow, L->d, L->W_w, L->d,
                       static_cast<float *>(P.wI) + (long long)b * n_loc * a.n_hI, a.n_hI, HCA_F32, n_loc, a.n_hI,
                       L->d, wscale, s);
      if (rc) return rc;
    }
  }
  // ---- window rows of the halo and the rank's tokens: [B, h + n_loc, c] at tokens t0 - h ..
  const int R = a.B * (h + n_loc);
  rc = launch_gemm(dt, H, L->d, L->W_KV, L->d, P.kv32, a.c, HCA_F32, R, a.c, L->d, 1.f, s);
  if (rc) return rc;
  {
    RowOpParams r{};
    r.in = static_cast<const float *>(P.kv32); r.in_stride = a.c; r.out = P.kvw; r.out_stride = a.c;
    r.out_dtype = dt; r.rows = R; r.cols = a.c; r.norm = 1; r.eps = eps; r.rd = a.rd; r.theta = theta;
    r.rows_per_pos = 1; r.pos_mod = h + n_loc; r.pos_base = t0 - h; r.scale = 1.f;
    if ((rc = launch_row_op(r, s))) return rc;
  }
  // ---- select and attend against the gathered caches (bf16 rows: the
  // stages exchange dtype entries even when the decode cache is mixed)
  hca_attn_desc ad = a;
  ad.kv_mixed = 0;
  if (csa) {
    rc = csa_index_topk(&ad, P.qI, static_cast<const float *>(P.wI), key_I, key_I_scale, cap, n_loc, t0,
                        static_cast<int32_t *>(P.idx), nullptr, 0, P.topk_ws, P.topk_bytes, stream);
    if (rc) return rc;
    return csa_attend(&ad, P.q, kv_comp, cap, static_cast<const int32_t *>(P.idx), P.kvw, 0, L->sink, n_loc, t0, o,
                      nullptr, 0, stream);
  }
  return hca_attend(&ad, P.q, kv_comp, cap, P.kvw, 0, L->sink, n_loc, t0, o, nullptr, 0, stream);
}

int hybrid_workspace_map(const hca_layer *L, int n, int decode, hca_ws_map *map) {
  int rc = check_layer(L);
  if (rc) return rc;
  if (!map) return fail(HCA_ERR_INVALID, "null map");
  if (n < (decode ? 1 : 0)) return fail(HCA_ERR_INVALID, "n must be >= %d", decode ? 1 : 0);
  const bool csa = L->kind == HCA_LAYER_CSA, comp = L->kind != HCA_LAYER_SWA;
  *map = hca_ws_map{-1, -1, -1, -1, -1, -1, -1};
  if (decode) {
    // hybrid_decode_step keeps the CSA index lists at the start of its workspace
    if (csa) map->idx = 0;
    return HCA_OK;
  }
  // plan against a stand-in base address and report the distances from it
  char *const base = reinterpret_cast<char *>(uintptr_t(1) << 40);
  Plan P{};
  plan_prefill(L, n, base, P);
  auto off = [&](void *p) -> long long { return p ? (long long)(static_cast<char *>(p) - base) : -1; };
  map->idx = csa ? off(P.idx) : -1;
  map->q = off(P.q);
  map->qI = csa ? off(P.qI) : -1;
  map->wI = csa ? off(P.wI) : -1;
  map->key_I = csa ? off(P.keyI) : -1;
  map->kv_comp = comp ? off(P.kvc) : -1;
  map->kv_win = off(P.kvw);
  return HCA_OK;
}

// ----------------------------------------------------------------- decode
// ---------------------------------------------------------------- decode inputs
// The projections of one decode token per sequence from hidden states
// h [B, d] at position pos, into the buffers of x (the same steps as the
// prefill's, with every row at position pos): [J] Eq.(9)-(10) / (20)-(21)
// compressor C/Z, Eq.(13) c^Q = RMSNorm(h W_DQ), Eq.(18) q = per-head RMSNorm
// of c^Q W_UQ then RoPE, the window row RMSNorm(h W_KV) then RoPE, and for CSA
// Eq.(14)-(15) q^I = RoPE(c^Q W_IUQ), w^I = h W_w c_I^-1/2 n_hI^-1/2, and the
// indexer compressor's C/Z.
struct DecPlan {
  void *cQ32, *cQ, *q32, *qI32, *kv32;
  size_t total;
};
static DecPlan plan_decode_inputs(const hca_layer *L, void *ws) {
  const hca_attn_desc &a = L->a;
  const bool csa = L->kind == HCA_LAYER_CSA;
  const long long T = a.B;
  Carver cv(ws);
  DecPlan P{};
  P.cQ32 = cv.take(T * L->d_c * 4);
  P.cQ = cv.take(T * L->d_c * esize(a.dtype));
  P.q32 = cv.take(T * a.n_h * a.c * 4);
  P.qI32 = csa ? cv.take(T * a.n_hI * a.c_I * 4) : nullptr;
  P.kv32 = cv.take(T * a.c * 4);
  P.total = cv.off;
  return P;
}

size_t hybrid_decode_inputs_workspace_size(const hca_layer *L) {
  if (check_layer(L)) return 0;
  return plan_decode_inputs(L, nullptr).total;
}

int hybrid_decode_inputs(const hca_layer *L, const void *h, int pos, const hca_token_in *x, void *ws,
                         size_t ws_bytes, hca_stream_t stream) {
  int rc = check_layer(L);
  if (rc) return rc;
  const hca_attn_desc &a = L->a;
  const bool csa = L->kind == HCA_LAYER_CSA, comp = L->kind != HCA_LAYER_SWA;
  if (!h || !x || pos < 0) return fail(HCA_ERR_INVALID, "h and x must be non-null and pos >= 0");
  if (!x->q || (a.w > 0 && !x->kv) || (comp && !x->comp) || (csa && (!x->qI || !x->wI || !x->compI)))
    return fail(HCA_ERR_INVALID, "missing output buffer in x");
  const DecPlan need = plan_decode_inputs(L, nullptr);
  if (ws_bytes < need.total || !ws) return fail(HCA_ERR_INVALID, "workspace too small");
  const DecPlan P = plan_decode_inputs(L, ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const hca_dtype dt = a.dtype;
  const float theta = rope_theta(a), eps = eps_of(a);
  const int T = a.B;
  auto row_op = [&](const void *in, int cols, void *out, hca_dtype odt, int rows, int norm, int rd,
                    int rows_per_pos) {
    RowOpParams r{};
    r.in = static_cast<const float *>(in); r.in_stride = cols; r.out = out; r.out_stride = cols; r.out_dtype = odt;
    r.rows = rows; r.cols = cols; r.norm = norm; r.eps = eps; r.rd = rd; r.theta = theta;
    r.rows_per_pos = rows_per_pos; r.pos_mod = 1; r.pos_base = pos; r.scale = 1.f;
    return launch_row_op(r, s);
  };
  void *q = const_cast<void *>(x->q);
  // compressor C/Z (fp32, [B, ncz c]: C_a | C_b | Z_a | Z_b, or C | Z)
  if (comp) {
    const int ncz = csa ? 4 : 2;
    rc = launch_gemm(dt, h, L->d, L->W_comp, L->d, const_cast<float *>(x->comp), (long long)ncz * a.c, HCA_F32, T,
                     ncz * a.c, L->d, 1.f, s);
    if (rc) return rc;
  }
  if (csa) {
    rc = launch_gemm(dt, h, L->d, L->W_compI, L->d, const_cast<float *>(x->compI), 4LL * a.c_I, HCA_F32, T,
                     4 * a.c_I, L->d, 1.f, s);
    if (rc) return rc;
  }
  // queries
  if ((rc = launch_gemm(dt, h, L->d, L->W_DQ, L->d, P.cQ32, L->d_c, HCA_F32, T, L->d_c, L->d, 1.f, s)) ||
      (rc = row_op(P.cQ32, L->d_c, P.cQ, dt, T, 1, 0, 1)))
    return rc;
  const int HC = a.n_h * a.c;
  if ((rc = launch_gemm(dt, P.cQ, L->d_c, L->W_UQ, L->d_c, P.q32, HC, HCA_F32, T, HC, L->d_c, 1.f, s)) ||
      (rc = row_op(P.q32, a.c, q, dt, T * a.n_h, 1, a.rd, a.n_h)))
    return rc;
  if (csa) {
    const int HI = a.n_hI * a.c_I;
    if ((rc = launch_gemm(dt, P.cQ, L->d_c, L->W_IUQ, L->d_c, P.qI32, HI, HCA_F32, T, HI, L->d_c, 1.f, s)) ||
        (rc = row_op(P.qI32, a.c_I, const_cast<void *>(x->qI), dt, T * a.n_hI, 0, a.rd_I, a.n_hI)))
      return rc;
    const float wscale = 1.0f / sqrtf((float)a.c_I) / sqrtf((float)a.n_hI);
    rc = launch_gemm(dt, h, L->d, L->W_w, L->d, const_cast<float *>(x->wI), a.n_hI, HCA_F32, T, a.n_hI, L->d, wscale,
                     s);
    if (rc) return rc;
  }
  // window row
  if (a.w > 0) {
    if ((rc = launch_gemm(dt, h, L->d, L->W_KV, L->d, P.kv32, a.c, HCA_F32, T, a.c, L->d, 1.f, s)) ||
        (rc = row_op(P.kv32, a.c, const_cast<void *>(x->kv), dt, T, 1, a.rd, 1)))
      return rc;
  }
  return HCA_OK;
}

size_t hybrid_decode_step_workspace_size(const hca_layer *L, int pos) {
  if (check_layer(L) || pos < 0) return 0;
  size_t b = 0;
  if (L->kind == HCA_LAYER_CSA) {
    b += (((size_t)L->a.B * L->a.k * 4) + 255) & ~(size_t)255;
    b += csa_index_topk_workspace_size(&L->a, 1, pos);
  }
  const size_t att = L->kind == HCA_LAYER_CSA ? csa_attend_workspace_size(&L->a, 1, pos)
                                              : hca_attend_workspace_size(&L->a, 1, pos);
  // mixed-precision KV: the emitted entry in bf16 before it is quantised
  const size_t mix = L->a.kv_mixed ? ((((size_t)L->a.B * L->a.c * 2) + 255) & ~(size_t)255) : 0;
  return ((b + 255) & ~(size_t)255) + att + 256 + mix;
}

int hybrid_decode_step(const hca_layer *L, const hca_token_in *x, hca_cache *cache, int pos, void *o, void *ws,
                       size_t ws_bytes, hca_stream_t stream) {
  int rc = check_layer(L);
  if (rc) return rc;
  const hca_attn_desc &a = L->a;
  const bool csa = L->kind == HCA_LAYER_CSA, comp = L->kind != HCA_LAYER_SWA;
  if (!x || !cache || !o || pos < 1) return fail(HCA_ERR_INVALID, "x, cache, o must be non-null and pos >= 1");
  if (!x->q || (a.w > 0 && (!x->kv || !cache->win)) || (comp && (!x->comp || !cache->kv_comp || !cache->state_kv)) ||
      (csa && (!x->qI || !x->wI || !x->compI || !cache->key_I || !cache->stateI_kv)))
    return fail(HCA_ERR_INVALID, "missing decode input or cache buffer");
  const int E = comp ? (pos + 1) / a.m : 0;
  if (comp && cache->cap < E) return fail(HCA_ERR_INVALID, "cache cap (%d) < entries (%d)", cache->cap, E);
  const size_t need = hybrid_decode_step_workspace_size(L, pos);
  if (ws_bytes < need || (need > 256 && !ws)) return fail(HCA_ERR_INVALID, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const hca_dtype dt = a.dtype;
  const float theta = rope_theta(a), eps = eps_of(a);
  void *mix_entry = a.kv_mixed ? static_cast<char *>(ws) + (need - ((((size_t)a.B * a.c * 2) + 255) & ~(size_t)255))
                               : nullptr;
  const int rec = a.kv_mixed ? (int)kv_mixed_row_bytes(a.c, a.rd) : 0;
  // 1. one launch: window ring write, compressor states (+ entry emission) of
  //    the main and (CSA) indexer compressors
  {
    CompressParams pm{}, pi{};
    if (comp) {
      hca_compress_desc cd{};
      cd.B = a.B; cd.width = a.c; cd.m = a.m; cd.overlap = csa ? a.overlap : 0; cd.rd = a.rd;
      cd.flags = HCA_COMPRESS_NORM | HCA_COMPRESS_ROPE; cd.eps = eps; cd.rope_theta = theta;
      cd.in_dtype = HCA_F32; cd.out_dtype = dt;
      const int ncz = csa ? 4 : 2;
      const float *cz = x->comp;
      const bool ov = cd.overlap != 0;
      rc = compress_params(&cd, pos, 1, cz, ov ? cz + a.c : nullptr, cz + (csa ? 2 : 1) * a.c, ov ? cz + 3 * a.c : nullptr,
                           (long long)ncz * a.c, (long long)ncz * a.c, L->B_comp, ov ? L->B_comp + a.m * a.c : nullptr,
                           nullptr, cache->kv_comp, nullptr, cache->cap, cache->state_kv, cache->state_score, &pm);
      if (rc) return rc;
      if (a.kv_mixed) {
        // mixed-precision KV: the emitted entry lands in a one-row bf16 scratch
        // per sequence (quantised into the cache below)
        pm.out = mix_entry;
        pm.out_seq_stride = 1;
        pm.e_first = pos / a.m;
      }
    }
    if (csa) {
      hca_compress_desc cd{};
      cd.B = a.B; cd.width = a.c_I; cd.m = a.m; cd.overlap = a.overlap; cd.rd = a.rd_I;
      cd.flags = HCA_COMPRESS_NORM | HCA_COMPRESS_ROPE; cd.eps = eps; cd.rope_theta = theta;
      cd.in_dtype = HCA_F32; cd.out_dtype = a.idx_key_dtype;
      const float *cz = x->compI;
      const bool ov = a.overlap != 0;
      rc = compress_params(&cd, pos, 1, cz, ov ? cz + a.c_I : nullptr, cz + 2 * a.c_I, ov ? cz + 3 * a.c_I : nullptr,
                           4LL * a.c_I, 4LL * a.c_I, L->B_compI, ov ? L->B_compI + a.m * a.c_I : nullptr, nullptr,
                           cache->key_I, cache->key_I_scale, cache->cap, cache->stateI_kv, cache->stateI_score, &pi);
      if (rc) return rc;
    }
    IngestRing ring{};
    if (a.w > 0 && !a.kv_mixed) {
      ring.row = x->kv; ring.ring = cache->win; ring.w = a.w; ring.c = a.c; ring.slot = pos % a.w; ring.dtype = dt;
    }
    if (comp || csa || ring.ring) {
      rc = launch_decode_ingest(comp ? &pm : nullptr, csa ? &pi : nullptr, ring, a.B, pos, s);
      if (rc) return rc;
    }
    if (a.kv_mixed) {
      // the token's window row and (on a block's last token) the new entry, as records
      if (a.w > 0) {
        rc = launch_kv_quant_mixed(x->kv, dt, a.B, a.c, a.rd, static_cast<char *>(cache->win) + (size_t)(pos % a.w) * rec,
                                   s, 1, a.w);
        if (rc) return rc;
      }
      if (comp && (pos + 1) % a.m == 0) {
        rc = launch_kv_quant_mixed(mix_entry, dt, a.B, a.c, a.rd,
                                   static_cast<char *>(cache->kv_comp) + (size_t)(pos / a.m) * rec, s, 1, cache->cap);
        if (rc) return rc;
      }
    }
  }
  if (csa) {
    char *w = static_cast<char *>(ws);
    int32_t *idx = reinterpret_cast<int32_t *>(w);
    const size_t ib = (((size_t)a.B * a.k * 4) + 255) & ~(size_t)255;
    const size_t tb = csa_index_topk_workspace_size(&a, 1, pos);
    rc = csa_index_topk(&a, x->qI, x->wI, cache->key_I, cache->key_I_scale, cache->cap, 1, pos, idx, nullptr, 0,
                        w + ib, tb, stream);
    if (rc) return rc;
    const size_t ab = (ib + tb + 255) & ~(size_t)255;
    return csa_attend(&a, x->q, cache->kv_comp, cache->cap, idx, cache->win, 1, L->sink, 1, pos, o, w + ab,
                      ws_bytes - ab, stream);
  }
  if (comp)
    return hca_attend(&a, x->q, cache->kv_comp, cache->cap, cache->win, 1, L->sink, 1, pos, o, ws, ws_bytes,
                      stream);
  hca_attn_desc ad = a;
  ad.m = pos + 2;
  return hca_attend(&ad, x->q, cache->win, 1, cache->win, 1, L->sink, 1, pos, o, nullptr, 0, stream);
}

}  // extern "C"
