// api.cu -- the extern "C" entry points of libhca: host-side validation,
// workspace carving and dispatch to the kernels.  See include/hca.h.
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace hca {

__device__ int g_status = 0;

static thread_local char t_err[512] = "";
static std::atomic<long long> g_launches{0};

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof t_err, fmt, ap);
  va_end(ap);
  return code;
}

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int check_launch(const char *what) {
  count_launch(1);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return HCA_OK;
}

// ---------------------------------------------------------------- profiler
namespace {
struct Pending { const char *name; cudaEvent_t a, b; };
std::mutex g_pm;
bool g_prof = false;
std::vector<Pending> g_pend;
std::vector<cudaEvent_t> g_free_events;
std::map<std::string, std::pair<double, long long>> g_acc;
cudaEvent_t take_event() {
  if (!g_free_events.empty()) {
    cudaEvent_t e = g_free_events.back();
    g_free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
// Inside a stream capture the record must be an external event node to be
// timeable after the graph is replayed.
void record_event(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else cudaEventRecord(e, s);
}
}  // namespace

LaunchScope::LaunchScope(const char *n, cudaStream_t s) : name(n), stream(s) {
  if (!g_prof) return;
  std::lock_guard<std::mutex> lk(g_pm);
  cudaEvent_t a = take_event();
  record_event(a, s);
  slot = (int)g_pend.size();
  g_pend.push_back({n, a, nullptr});
}

int LaunchScope::done() {
  if (slot >= 0) {
    std::lock_guard<std::mutex> lk(g_pm);
    cudaEvent_t b = take_event();
    record_event(b, stream);
    if (slot < (int)g_pend.size()) g_pend[slot].b = b;
  }
  return check_launch(name);
}

int *device_status_ptr() {
  static std::atomic<int *> ptr[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!ptr[dev]) {
    void *a = nullptr;
    if (cudaGetSymbolAddress(&a, g_status) == cudaSuccess) ptr[dev] = static_cast<int *>(a);
  }
  return ptr[dev];
}

int encode_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                   uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess || !fn)
      return fail(HCA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HCA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return HCA_OK;
}

int device_slot() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return 0;
  }
  return dev;
}

int num_sms() {
  static std::atomic<int> n[kMaxDevices];
  const int d = device_slot();
  if (n[d] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || v <= 0) {
      (void)cudaGetLastError();
      v = 148;
    }
    n[d] = v;
  }
  return n[d];
}

namespace {

size_t esize(hca_dtype t) { return t == HCA_F32 ? 4 : ((t == HCA_BF16 || t == HCA_FP4) ? 2 : 1); }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

#define REQUIRE(cond, ...)                                   \
  do {                                                       \
    if (!(cond)) return fail(HCA_ERR_INVALID, __VA_ARGS__);  \
  } while (0)

int check_attn_desc(const hca_attn_desc *d, bool need_indexer) {
  REQUIRE(d != nullptr, "null descriptor");
  REQUIRE(d->B >= 1, "B must be >= 1 (got %d)", d->B);
  REQUIRE(d->n_h >= 1, "n_h must be >= 1");
  REQUIRE(d->c >= 32 && d->c <= 512 && d->c % 32 == 0, "c must be a multiple of 32 in [32, 512] (got %d)", d->c);
  REQUIRE(d->rd >= 0 && d->rd <= d->c && d->rd % 2 == 0, "rd must be even and <= c");
  REQUIRE(d->w >= 0, "w must be >= 0");
  REQUIRE(d->m >= 1, "m must be >= 1");
  REQUIRE(d->dtype == HCA_F32 || d->dtype == HCA_BF16, "dtype must be HCA_F32 or HCA_BF16");
  REQUIRE(d->max_ctas >= 0, "max_ctas must be >= 0 (0 = every SM)");
  REQUIRE(d->kv_mixed == 0 || d->kv_mixed == 1, "kv_mixed must be 0 or 1");
  if (d->kv_mixed) {
    REQUIRE(d->dtype == HCA_BF16, "mixed-precision KV rows need dtype HCA_BF16");
    REQUIRE(kv_mixed_row_bytes(d->c, d->rd) > 0, "mixed-precision KV rows need c - rd a multiple of 64 and rd a "
            "multiple of 16 (c = %d, rd = %d)", d->c, d->rd);
  }
  if (need_indexer) {
    REQUIRE(d->k >= 1, "k must be >= 1");
    REQUIRE(d->n_hI >= 1 && d->c_I >= 8 && d->c_I % 8 == 0, "indexer heads / dim invalid");
    REQUIRE(d->rd_I >= 0 && d->rd_I <= d->c_I && d->rd_I % 2 == 0, "rd_I must be even and <= c_I");
    REQUIRE(d->idx_key_dtype == HCA_F32 || d->idx_key_dtype == HCA_BF16 || d->idx_key_dtype == HCA_FP8E4M3 ||
                d->idx_key_dtype == HCA_FP4,
            "idx_key_dtype invalid");
    REQUIRE(d->idx_key_dtype != HCA_FP4 || d->c_I == 64, "the FP4 indexer path needs c_I == 64");
  }
  return HCA_OK;
}

float attn_scale(const hca_attn_desc *d) { return d->scale > 0.f ? d->scale : 1.0f / sqrtf((float)d->c); }

IndexParams index_params(const hca_attn_desc *d, const void *qI, const float *wI, const void *KI,
                         const float *KI_scale, int cap, int n_q, int start_pos) {
  IndexParams p{};
  p.B = d->B; p.n_q = n_q; p.start_pos = start_pos; p.m = d->m; p.n_hI = d->n_hI; p.c_I = d->c_I;
  p.cap = cap; p.k = d->k; p.qI = qI; p.wI = wI; p.KI = KI; p.KI_scale = KI_scale;
  p.q_dtype = d->dtype; p.key_dtype = d->idx_key_dtype;
  p.status = device_status_ptr();
  return p;
}

AttendParams attend_params(const hca_attn_desc *d, const void *q, const void *kv_comp, int cap,
                           const int32_t *idx, const void *kv_win, int win_is_ring, const float *sink,
                           int n_q, int start_pos, void *o, int csa) {
  AttendParams p{};
  p.B = d->B; p.n_q = n_q; p.start_pos = start_pos; p.n_h = d->n_h; p.c = d->c; p.rd = d->rd;
  p.w = d->w; p.m = d->m; p.k = csa ? d->k : 0; p.cap = cap; p.csa = csa; p.win_is_ring = win_is_ring;
  p.scale = attn_scale(d); p.theta = d->rope_theta > 0.f ? d->rope_theta : 10000.f;
  p.kv_mixed = d->kv_mixed ? 1 : 0;
  p.rec = d->kv_mixed ? (int)kv_mixed_row_bytes(d->c, d->rd) : 0;
  p.q = q; p.kv_comp = kv_comp; p.idx = idx; p.kv_win = kv_win; p.sink = sink; p.o = o; p.dtype = d->dtype;
  // token-indexed window: the rows of tokens start_pos - h .. start_pos + n_q - 1,
  // h = min(w - 1, start_pos) (the halo before the first query)
  const int halo = d->w > 0 ? (d->w - 1 < start_pos ? d->w - 1 : start_pos) : 0;
  p.win_tok0 = start_pos - halo;
  p.win_rows = n_q + halo;
  p.status = nullptr;
  p.nsplit = 1;
  p.cluster = 0;
  p.max_ctas = d->max_ctas;
  return p;
}

int check_attend_args(const hca_attn_desc *d, const void *q, const void *kv_comp, int cap, const void *kv_win,
                      int win_is_ring, const float *sink, int n_q, int start_pos, const void *o) {
  REQUIRE(n_q >= 0 && start_pos >= 0, "n_q and start_pos must be >= 0");
  REQUIRE(q && o && sink, "q, sink and o must be non-null");
  REQUIRE(aligned16(q) && aligned16(o), "q and o must be 16-byte aligned");
  const int vmax = (start_pos + n_q) / d->m;
  REQUIRE(cap >= vmax, "cap (%d) < visible entries (%d)", cap, vmax);
  REQUIRE(vmax == 0 || (kv_comp && aligned16(kv_comp)), "kv_comp must be non-null and 16-byte aligned");
  if (d->w > 0) REQUIRE(kv_win && aligned16(kv_win), "kv_win must be non-null and 16-byte aligned");
  if (win_is_ring) REQUIRE(n_q <= 1, "a ring window serves one query per sequence");
  return HCA_OK;
}

}  // namespace
int compress_params(const hca_compress_desc *d, int start_pos, int n, const void *Ca, const void *Cb,
                    const void *Za, const void *Zb, long long row_stride, long long seq_stride, const float *Ba,
                    const float *Bb, const float *gamma, void *out, float *out_scale, long long out_seq_stride,
                    float *state_kv, float *state_score, CompressParams *pp) {
  REQUIRE(d != nullptr, "null descriptor");
  REQUIRE(d->B >= 1 && d->m >= 1, "B and m must be >= 1");
  REQUIRE(d->width >= 8 && d->width % 8 == 0, "width must be a positive multiple of 8");
  REQUIRE(d->overlap == 0 || d->overlap == 1, "overlap must be 0 or 1");
  REQUIRE(d->in_dtype == HCA_F32 || d->in_dtype == HCA_BF16, "in_dtype must be f32 or bf16");
  REQUIRE(d->out_dtype == HCA_F32 || d->out_dtype == HCA_BF16 || d->out_dtype == HCA_FP8E4M3 ||
              d->out_dtype == HCA_FP4, "bad out_dtype");
  REQUIRE(d->out_dtype != HCA_FP4 || d->width == 64, "FP4 entries need width 64");
  if (d->flags & HCA_COMPRESS_ROPE)
    REQUIRE(d->rd >= 0 && d->rd <= d->width && d->rd % 8 == 0, "rd must be a multiple of 8 and <= width");
  REQUIRE(n >= 0 && start_pos >= 0, "n and start_pos must be >= 0");
  REQUIRE(Ca && Za && Ba, "Ca, Za and Ba must be non-null");
  if (d->overlap) REQUIRE(Cb && Zb && Bb, "overlap needs Cb, Zb and Bb");
  const size_t es = esize(d->in_dtype);
  REQUIRE(aligned16(Ca) && aligned16(Za) && (!d->overlap || (aligned16(Cb) && aligned16(Zb))),
          "C/Z pointers must be 16-byte aligned");
  REQUIRE(row_stride >= d->width && (row_stride * (long long)es) % 16 == 0, "row_stride invalid");
  REQUIRE((seq_stride * (long long)es) % 16 == 0, "seq_stride must keep 16-byte alignment");
  REQUIRE(d->out_dtype != HCA_FP8E4M3 || out_scale, "fp8 output needs out_scale");
  if (start_pos > 0) {
    REQUIRE(n == 1, "decode mode (start_pos > 0) takes exactly one token");
    REQUIRE(state_kv && state_score, "decode mode needs the compressor state");
    if ((start_pos + 1) % d->m == 0)
      REQUIRE(out && aligned16(out) && out_seq_stride > start_pos / d->m, "out too small for entry %d",
              start_pos / d->m);
  }
  CompressParams p{};
  p.B = d->B; p.n = n; p.width = d->width; p.m = d->m; p.overlap = d->overlap;
  p.rd = (d->flags & HCA_COMPRESS_ROPE) ? d->rd : 0; p.flags = d->flags;
  p.eps = d->eps > 0.f ? d->eps : 1e-6f; p.theta = d->rope_theta > 0.f ? d->rope_theta : 10000.f;
  fill_rope_freq(p.rope_freq, (d->flags & HCA_COMPRESS_ROPE) ? d->rd : 0, p.theta);
  p.Ca = Ca; p.Cb = Cb; p.Za = Za; p.Zb = Zb; p.row_stride = row_stride; p.seq_stride = seq_stride;
  p.Ba = Ba; p.Bb = Bb; p.gamma = gamma; p.out = out; p.out_scale = out_scale; p.out_seq_stride = out_seq_stride;
  p.state_kv = state_kv; p.state_score = state_score; p.in_dtype = d->in_dtype; p.out_dtype = d->out_dtype;
  *pp = p;
  return HCA_OK;
}

// Failure-detection self-test: one thread waits on an mbarrier that nothing
// ever arrives on; the wait gives up after limit_ns, sets the status word to
// HCA_ERR_TIMEOUT and the kernel returns like any expired production wait.
__global__ void selftest_wait_kernel(unsigned long long limit_ns, int *status) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  mbar_fence_init();
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(b, 0)) return;   // cannot happen: nothing arrives
    if ((it & 255u) == 0 && global_ns() - t0 > limit_ns) {
      set_timeout_status(status);
      return;
    }
  }
}

}  // namespace hca

using namespace hca;

extern "C" {

const char *hca_last_error(void) { return t_err; }

int hca_version(void) { return (0 << 16) | 2; }

size_t hca_static_scratch_bytes(void) { return (size_t)HCA_STATIC_SCRATCH_BYTES; }

long long hca_launch_count(void) { return g_launches.load(); }

int hca_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_pm);
  g_prof = on != 0;
  return HCA_OK;
}

int hca_profile_sample(void) {
  std::lock_guard<std::mutex> lk(g_pm);
  for (auto &p : g_pend) {
    if (!p.b) continue;
    if (cudaEventSynchronize(p.b) != cudaSuccess) return fail(HCA_ERR_CUDA, "profile event sync failed");
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
      auto &acc = g_acc[p.name];
      acc.first += ms;
      acc.second += 1;
    }
  }
  return HCA_OK;
}

int hca_profile_collect(char *buf, size_t len) {
  std::lock_guard<std::mutex> lk(g_pm);
  if (!buf || len == 0) return fail(HCA_ERR_INVALID, "null profile buffer");
  size_t off = 0;
  buf[0] = 0;
  for (auto &kv : g_acc) {
    const int w = snprintf(buf + off, len - off, "%s\t%lld\t%.6f\n", kv.first.c_str(), kv.second.second,
                           kv.second.first);
    if (w < 0 || (size_t)w >= len - off) return fail(HCA_ERR_INVALID, "profile buffer too small");
    off += (size_t)w;
  }
  g_acc.clear();
  for (auto &p : g_pend) {
    if (p.b) g_free_events.push_back(p.b);
    g_free_events.push_back(p.a);
  }
  g_pend.clear();
  return HCA_OK;
}

int hca_selftest_wait(unsigned long long limit_ns, hca_stream_t stream) {
  REQUIRE(limit_ns >= 1000000ull && limit_ns <= kWaitLimitNs, "limit_ns must be within [1 ms, 2 s]");
  int *status = device_status_ptr();
  REQUIRE(status != nullptr, "no device status word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return HCA_LAUNCH("selftest_wait", s, selftest_wait_kernel<<<1, 32, 0, s>>>(limit_ns, status));
}

int hca_check_status(hca_stream_t stream, int *device_status) {
  if (!device_status) return fail(HCA_ERR_INVALID, "null device_status");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof v);
  if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  const int zero = 0;
  cudaMemcpyToSymbol(g_status, &zero, sizeof zero);
  *device_status = v;
  return HCA_OK;
}

// ----------------------------------------------------------------- compress
int csa_compress(const hca_compress_desc *d, int start_pos, int n, const void *Ca, const void *Cb,
                 const void *Za, const void *Zb, long long row_stride, long long seq_stride,
                 const float *Ba, const float *Bb, const float *gamma, void *out, float *out_scale,
                 long long out_seq_stride, float *state_kv, float *state_score, hca_stream_t stream) {
  CompressParams p{};
  int rc = compress_params(d, start_pos, n, Ca, Cb, Za, Zb, row_stride, seq_stride, Ba, Bb, gamma, out, out_scale,
                           out_seq_stride, state_kv, state_score, &p);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (start_pos == 0) {
    const int E = n / d->m;
    if (E > 0) {
      REQUIRE(out && aligned16(out) && out_seq_stride >= E, "out must hold n/m entries per sequence");
      rc = launch_compress_prefill(p, s);
      if (rc) return rc;
    }
    if (state_kv || state_score) {
      REQUIRE(state_kv && state_score, "state_kv and state_score go together");
      return launch_compress_state_prefill(p, s);
    }
    return HCA_OK;
  }
  return launch_compress_decode(p, start_pos, s);
}

int hca_compress(const hca_compress_desc *d, int start_pos, int n, const void *Ca, const void *Cb,
                 const void *Za, const void *Zb, long long row_stride, long long seq_stride,
                 const float *Ba, const float *Bb, const float *gamma, void *out, float *out_scale,
                 long long out_seq_stride, float *state_kv, float *state_score, hca_stream_t stream) {
  return csa_compress(d, start_pos, n, Ca, Cb, Za, Zb, row_stride, seq_stride, Ba, Bb, gamma, out, out_scale,
                      out_seq_stride, state_kv, state_score, stream);
}

// ----------------------------------------------------------------- index + top-k
size_t csa_index_topk_workspace_size(const hca_attn_desc *d, int n_q, int start_pos) {
  if (!d || d->m < 1 || n_q < 0 || start_pos < 0) return 0;
  IndexParams p = index_params(d, nullptr, nullptr, nullptr, nullptr, 0, n_q, start_pos);
  return topk_workspace_bytes(p);
}

int csa_index_topk(const hca_attn_desc *d, const void *qI, const float *wI, const void *KI,
                   const float *KI_scale, int cap, int n_q, int start_pos, int32_t *idx, float *scores,
                   long long score_stride, void *ws, size_t ws_bytes, hca_stream_t stream) {
  int rc = check_attn_desc(d, true);
  if (rc) return rc;
  REQUIRE(n_q >= 0 && start_pos >= 0, "n_q and start_pos must be >= 0");
  REQUIRE(qI && wI && idx, "qI, wI and idx must be non-null");
  const int vmax = (start_pos + n_q) / d->m;
  REQUIRE(cap >= vmax, "cap (%d) < visible entries (%d)", cap, vmax);
  REQUIRE(vmax == 0 || KI, "KI must be non-null");
  REQUIRE(d->idx_key_dtype != HCA_FP8E4M3 || KI_scale, "fp8 keys need KI_scale");
  if (scores) REQUIRE(score_stride >= vmax, "score_stride < max visible entries");
  IndexParams p = index_params(d, qI, wI, KI, KI_scale, cap, n_q, start_pos);
  REQUIRE(ws || topk_workspace_bytes(p) == 0, "workspace required");
  return run_index_topk(p, idx, scores, score_stride, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int csa_index_topk_static_scratch(const hca_attn_desc *d, const void *qI, const float *wI, const void *KI,
                                  const float *KI_scale, int cap, int n_q, int start_pos, int32_t *idx,
                                  float *scores, long long score_stride, hca_stream_t stream) {
  int rc = check_attn_desc(d, true);
  if (rc) return rc;
  REQUIRE(n_q >= 0 && start_pos >= 0, "n_q and start_pos must be >= 0");
  REQUIRE(qI && wI && idx, "qI, wI and idx must be non-null");
  const int vmax = (start_pos + n_q) / d->m;
  REQUIRE(cap >= vmax, "cap (%d) < visible entries (%d)", cap, vmax);
  REQUIRE(vmax == 0 || KI, "KI must be non-null");
  REQUIRE(d->idx_key_dtype != HCA_FP8E4M3 || KI_scale, "fp8 keys need KI_scale");
  if (scores) REQUIRE(score_stride >= vmax, "score_stride < max visible entries");
  IndexParams p = index_params(d, qI, wI, KI, KI_scale, cap, n_q, start_pos);
  return run_index_topk_static(p, idx, scores, score_stride, static_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------- output projection
size_t hca_output_projection_workspace_size(const hca_oproj_desc *d) {
  if (!d || d->T < 0 || d->g < 1 || d->d_g < 1) return 0;
  const size_t b = (size_t)d->T * d->g * d->d_g * esize(d->dtype);
  return (b + 255) & ~(size_t)255;
}

int hca_output_projection(const hca_oproj_desc *d, const void *o, const void *wo_a, const void *wo_b, void *out,
                          void *ws, size_t ws_bytes, hca_stream_t stream) {
  REQUIRE(d != nullptr, "null descriptor");
  REQUIRE(d->T >= 0 && d->n_h >= 1 && d->c >= 1 && d->g >= 1 && d->d_g >= 1 && d->d >= 1, "bad shape");
  REQUIRE(d->n_h % d->g == 0, "n_h (%d) must be a multiple of g (%d)", d->n_h, d->g);
  REQUIRE(d->dtype == HCA_F32 || d->dtype == HCA_BF16, "dtype must be f32 or bf16");
  REQUIRE(d->out_dtype == HCA_F32 || d->out_dtype == HCA_BF16, "out_dtype must be f32 or bf16");
  if (d->T == 0) return HCA_OK;
  REQUIRE(o && wo_a && wo_b && out, "o, wo_a, wo_b and out must be non-null");
  REQUIRE(aligned16(o) && aligned16(wo_a) && aligned16(wo_b) && aligned16(out), "pointers must be 16-byte aligned");
  REQUIRE(ws && ws_bytes >= hca_output_projection_workspace_size(d), "workspace too small");
  const int gw = d->n_h / d->g * d->c;          // values per group
  const int mid_n = d->g * d->d_g;
  const size_t es = esize(d->dtype);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const char *ob = static_cast<const char *>(o);
  const char *wa = static_cast<const char *>(wo_a);
  char *mid = static_cast<char *>(ws);
  for (int i = 0; i < d->g; ++i) {
    const int rc = launch_gemm(d->dtype, ob + (size_t)i * gw * es, (long long)d->n_h * d->c,
                               wa + (size_t)i * d->d_g * gw * es, gw, mid + (size_t)i * d->d_g * es, mid_n, d->dtype,
                               d->T, d->d_g, gw, 1.f, s);
    if (rc) return rc;
  }
  return launch_gemm(d->dtype, mid, mid_n, wo_b, mid_n, out, d->d, d->out_dtype, d->T, d->d, mid_n, 1.f, s);
}

// ------------------------------------------------------------ FP4 indexer
int hca_fp4_rotate_quant(const void *x, hca_dtype x_dtype, long long rows, int n, void *out, hca_stream_t stream) {
  REQUIRE(n == 64, "n must be 64 (the indexer head dim), got %d", n);
  REQUIRE(rows >= 0, "rows must be >= 0");
  REQUIRE(x_dtype == HCA_F32 || x_dtype == HCA_BF16, "x_dtype must be HCA_F32 or HCA_BF16");
  if (rows == 0) return HCA_OK;
  REQUIRE(x && out, "x and out must be non-null");
  REQUIRE(aligned16(x) && aligned16(out), "x and out must be 16-byte aligned");
  return launch_fp4_rotate_quant(x, x_dtype, rows, out, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------- step trace
int hca_step_trace(void *buf, size_t bytes) {
  REQUIRE(buf == nullptr || ((reinterpret_cast<uintptr_t>(buf) & 7u) == 0 && bytes >= 40),
          "buf must be 8-byte aligned and hold the counter and at least one record (40 bytes)");
  const unsigned long long cap = buf ? (unsigned long long)((bytes - 8) / 32) : 0ull;
  int rc = step_trace_set_attend(buf, cap);
  if (!rc) rc = step_trace_set_index_tc(buf, cap);
  if (!rc) rc = step_trace_set_index_topk(buf, cap);
  if (!rc) rc = step_trace_set_compress(buf, cap);
  if (rc) return fail(rc, "could not set the step trace buffer");
  return HCA_OK;
}

// ------------------------------------------------------ mixed-precision KV
size_t hca_kv_mixed_row_bytes(int c, int rd) { return kv_mixed_row_bytes(c, rd); }

int hca_kv_quant_mixed(const void *x, hca_dtype x_dtype, long long rows, int c, int rd, void *out,
                       hca_stream_t stream) {
  REQUIRE(kv_mixed_row_bytes(c, rd) > 0, "unsupported (c, rd) = (%d, %d): need c <= 512, rd %% 16 == 0, "
          "(c - rd) %% 64 == 0", c, rd);
  REQUIRE(rows >= 0, "rows must be >= 0");
  REQUIRE(x_dtype == HCA_F32 || x_dtype == HCA_BF16, "x_dtype must be HCA_F32 or HCA_BF16");
  if (rows == 0) return HCA_OK;
  REQUIRE(x && out, "x and out must be non-null");
  REQUIRE(aligned16(x) && aligned16(out), "x and out must be 16-byte aligned");
  return launch_kv_quant_mixed(x, x_dtype, rows, c, rd, out, static_cast<cudaStream_t>(stream));
}

int hca_kv_dequant_mixed(const void *in, long long rows, int c, int rd, void *out, hca_stream_t stream) {
  REQUIRE(kv_mixed_row_bytes(c, rd) > 0, "unsupported (c, rd) = (%d, %d): need c <= 512, rd %% 16 == 0, "
          "(c - rd) %% 64 == 0", c, rd);
  REQUIRE(rows >= 0, "rows must be >= 0");
  if (rows == 0) return HCA_OK;
  REQUIRE(in && out, "in and out must be non-null");
  REQUIRE(aligned16(in) && aligned16(out), "in and out must be 16-byte aligned");
  return launch_kv_dequant_mixed(in, rows, c, rd, out, static_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------- attend
size_t csa_attend_workspace_size(const hca_attn_desc *d, int n_q, int start_pos) {
  if (!d) return 0;
  AttendParams p = attend_params(d, nullptr, nullptr, 0, nullptr, nullptr, 0, nullptr, n_q, start_pos, nullptr, 1);
  return attend_workspace_bytes(p);
}
size_t hca_attend_workspace_size(const hca_attn_desc *d, int n_q, int start_pos) {
  if (!d) return 0;
  AttendParams p = attend_params(d, nullptr, nullptr, 0, nullptr, nullptr, 0, nullptr, n_q, start_pos, nullptr, 0);
  return attend_workspace_bytes(p);
}

int csa_attend(const hca_attn_desc *d, const void *q, const void *kv_comp, int cap, const int32_t *idx,
               const void *kv_win, int win_is_ring, const float *sink, int n_q, int start_pos, void *o,
               void *ws, size_t ws_bytes, hca_stream_t stream) {
  int rc = check_attn_desc(d, false);
  if (rc) return rc;
  REQUIRE(d->k >= 1, "k must be >= 1");
  rc = check_attend_args(d, q, kv_comp, cap, kv_win, win_is_ring, sink, n_q, start_pos, o);
  if (rc) return rc;
  REQUIRE(idx || n_q == 0, "idx must be non-null");
  AttendParams p = attend_params(d, q, kv_comp, cap, idx, kv_win, win_is_ring, sink, n_q, start_pos, o, 1);
  p.status = device_status_ptr();
  return run_attend(p, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int hca_attend(const hca_attn_desc *d, const void *q, const void *kv_comp, int cap, const void *kv_win,
               int win_is_ring, const float *sink, int n_q, int start_pos, void *o, void *ws, size_t ws_bytes,
               hca_stream_t stream) {
  int rc = check_attn_desc(d, false);
  if (rc) return rc;
  rc = check_attend_args(d, q, kv_comp, cap, kv_win, win_is_ring, sink, n_q, start_pos, o);
  if (rc) return rc;
  AttendParams p = attend_params(d, q, kv_comp, cap, nullptr, kv_win, win_is_ring, sink, n_q, start_pos, o, 0);
  p.status = device_status_ptr();
  return run_attend(p, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
