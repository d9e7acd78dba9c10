// internal.h -- host-side declarations shared by the libhca translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <cmath>

#include "../../include/hca.h"

namespace hca {

// Per-kernel timing with CUDA events on the launching stream (off unless
// hca_profile_enable(1) was called).  Usage:
//   return HCA_LAUNCH("name", stream, kernel<<<grid, block, smem, stream>>>(args));
struct LaunchScope {
  int slot = -1;
  const char *name;
  cudaStream_t stream;
  LaunchScope(const char *name, cudaStream_t s);
  int done();
};
#define HCA_LAUNCH(name, stream, ...) \
  ([&]() -> int { ::hca::LaunchScope _ls((name), (stream)); __VA_ARGS__; return _ls.done(); }())

// Record an error message for hca_last_error() and return `code`.
int fail(int code, const char *fmt, ...);
// Map a CUDA error after a launch; counts launches.
int check_launch(const char *what);
void count_launch(int n = 1);
int num_sms();
// The current device's slot in per-device caches (0 .. kMaxDevices-1; 0 when
// the device cannot be read).  Kernel attributes, occupancy figures and the SM
// count are cached per device, so one process may drive several devices.
constexpr int kMaxDevices = 64;
int device_slot();
// Encode a 2-D tiled TMA descriptor over a row-major matrix (rows x cols
// elements of elem_bytes, rows row_stride_bytes apart); box = box_rows x
// box_cols elements.  Returns HCA_OK or HCA_ERR_CUDA.
int encode_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dt, uint64_t cols,
                   uint64_t rows, uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows,
                   CUtensorMapSwizzle swizzle);
// Device address of the status word (HCA_OK or HCA_ERR_TIMEOUT) of the current device.
int *device_status_ptr();

// ------------------------------------------------------------- compress
// theta^(-2i/rd) for the first min(rd/2, 32) rotated pairs (host-computed).
inline void fill_rope_freq(double (&f)[32], int rd, float theta) {
  for (int i = 0; i < 32; ++i)
    f[i] = (rd > 0 && i < rd / 2) ? std::exp2(-2.0 * i / (double)rd * std::log2((double)theta)) : 0.0;
}

struct CompressParams {
  int B, n, width, m, overlap, rd, flags;
  float eps, theta;
  double rope_freq[32];    // fill_rope_freq(rd, theta)
  const void *Ca, *Cb, *Za, *Zb;
  long long row_stride, seq_stride;
  const float *Ba, *Bb, *gamma;
  void *out;
  float *out_scale;
  long long out_seq_stride;
  float *state_kv, *state_score;
  hca_dtype in_dtype, out_dtype;
  // prefill of a token range: local entries below e_first only feed the next
  // entry's b series and are not written (entry e goes to out slot e - e_first);
  // entry e sits at RoPE position (e_pos0 + e) * m
  long long e_first, e_pos0;
};
int launch_compress_prefill(const CompressParams &p, cudaStream_t s);
int launch_compress_state_prefill(const CompressParams &p, cudaStream_t s);
int launch_compress_decode(const CompressParams &p, int pos, cudaStream_t s);
// Validate a compressor call and fill its parameters (no launch).
int compress_params(const hca_compress_desc *d, int start_pos, int n, const void *Ca, const void *Cb,
                    const void *Za, const void *Zb, long long row_stride, long long seq_stride, const float *Ba,
                    const float *Bb, const float *gamma, void *out, float *out_scale, long long out_seq_stride,
                    float *state_kv, float *state_score, CompressParams *p);
// Window ring write of one decode token: row [B, c] -> ring[b, slot] of [B, w, c].
struct IngestRing {
  const void *row;
  void *ring;
  int w, c, slot;
  hca_dtype dtype;
};
// One launch per decode token of a layer: main compressor (pa, may be NULL),
// indexer compressor (pb, may be NULL) and the ring write (ring.ring may be NULL).
int launch_decode_ingest(const CompressParams *pa, const CompressParams *pb, const IngestRing &ring, int B, int pos,
                         cudaStream_t s);

// ------------------------------------------------------------- index + top-k
struct IndexParams {
  int B, n_q, start_pos, m, n_hI, c_I, cap, k;
  const void *qI;          // [B, n_q, n_hI, c_I]
  const float *wI;         // [B, n_q, n_hI]
  const void *KI;          // [B, cap, c_I]
  const float *KI_scale;   // [B, cap] fp8 only
  hca_dtype q_dtype, key_dtype;
  float *scores;           // [B, n_q, score_stride]
  long long score_stride;
  int *status;
  int round_bf16;          // FP4 path: scores rounded to bf16 (nearest even) when written
};
int launch_index_scores(const IndexParams &p, cudaStream_t s);
// tcgen05 scorer; returns HCA_ERR_UNSUPPORTED (launching nothing) for shapes it does not cover.
int launch_index_scores_tc(const IndexParams &p, cudaStream_t s);

struct TopkParams {
  int rows;                // number of score rows
  int k;
  const float *scores;     // fp32 scores, row r at scores + r*in_stride; or
  const uint32_t *keys;    // order keys (0 = absent) whose indices are in cand_idx
  const int32_t *cand_idx; // same layout as keys
  long long in_stride;
  int fixed_len;           // > 0: every row has fixed_len elements
  int n_q, start_pos, m;   // else row r -> query r % n_q at position start_pos + r % n_q, (t+1)/m entries
  int32_t *idx_out;        // (row, segment) at idx_out + row*out_stride + segment*k
  uint32_t *key_out;       // optional: the winners' order keys (segmented first pass)
  long long out_stride;
  int n_seg, seg_len, slice;   // segments per row, keys per segment, keys per CTA
};
size_t topk_workspace_bytes(const IndexParams &p);
int run_index_topk(const IndexParams &p, int32_t *idx, float *user_scores, long long user_stride,
                   void *ws, size_t ws_bytes, cudaStream_t s);
// csa_index_topk with its scratch in a file-scope device array of
// HCA_STATIC_SCRATCH_BYTES; fails with HCA_ERR_INVALID when the call needs more.
int run_index_topk_static(const IndexParams &p, int32_t *idx, float *user_scores, long long user_stride,
                          cudaStream_t s);

// ------------------------------------------------------------ FP4 indexer
// Rows of 64: Hadamard rotation, FP4 blocks of 32, written as exact bf16 values.
// Strided rows: row r at (r / per_seq) * seq_rows + r % per_seq (per_seq <= 0: dense).
int launch_fp4_rotate_quant(const void *x, hca_dtype dt, long long rows, void *out, cudaStream_t s,
                            long long per_seq = 0, long long seq_rows = 0);
// ------------------------------------------------------------- step trace
// Point the traced kernels of each translation unit at a record buffer (NULL = off).
int step_trace_set_attend(void *buf, unsigned long long cap);
int step_trace_set_index_tc(void *buf, unsigned long long cap);
int step_trace_set_index_topk(void *buf, unsigned long long cap);
int step_trace_set_compress(void *buf, unsigned long long cap);

// ------------------------------------------------------- mixed-precision KV
// Record bytes of one row (0 for unsupported shapes) and the two HBM streams.
size_t kv_mixed_row_bytes(int c, int rd);
// Output row r at record (r / per_seq) * seq_rows + r % per_seq (per_seq <= 0: dense).
int launch_kv_quant_mixed(const void *x, hca_dtype dt, long long rows, int c, int rd, void *out, cudaStream_t s,
                          long long per_seq = 0, long long seq_rows = 0);
int launch_kv_dequant_mixed(const void *in, long long rows, int c, int rd, void *out, cudaStream_t s);

// ------------------------------------------------------------- attention
// Division of dividends below 2^31 by an invariant divisor d >= 1 with one
// multiply-high, an add and a shift (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994): s = ceil(log2 d),
// mul = floor(2^32 (2^s - d) / d) + 1, n / d = (umulhi(n, mul) + n) >> s.
struct FastDiv {
  uint32_t mul, s;
};
inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  FastDiv f;
  f.mul = (uint32_t)((((1ull << 32) * ((1ull << s) - d)) / d) + 1);
  f.s = s;
  return f;
}
#ifdef __CUDACC__
__device__ __forceinline__ int fdiv(int n, const FastDiv &f) {
  return (int)((__umulhi((uint32_t)n, f.mul) + (uint32_t)n) >> f.s);
}
#endif

struct AttendParams {
  int B, n_q, start_pos, n_h, c, rd, w, m, k, cap;
  int csa;                 // 1: compressed set from idx; 0: all visible entries
  int win_is_ring;
  float scale, theta, sink_log2_bias;
  double rope_freq[32];    // theta^(-2i/rd) for the rd/2 rotated pairs (host-computed)
  const void *q;           // [B, n_q, n_h, c]
  const void *kv_comp;     // [B, cap, c]
  const int32_t *idx;      // [B, n_q, k]
  const void *kv_win;      // token rows [B, win_rows, c] (row r = token win_tok0 + r); ring [B, w, c]
  int win_tok0, win_rows;  // token-indexed window: first token and rows per sequence
  int kv_mixed;            // 1: kv_comp and kv_win hold mixed-precision records of `rec` bytes
  int rec;
  const float *sink;       // [n_h]
  void *o;                 // [B, n_q, n_h, c]
  hca_dtype dtype;
  int *status;
  // split-KV: each query's key list is cut into nsplit tile ranges whose
  // unnormalised partials (fp32 O rows, running max and sum) are merged
  // either by the CTAs of one thread-block cluster through distributed shared
  // memory (cluster = 1, nsplit <= 8) or through part_o / part_ml and a
  // combine kernel (cluster = 0)
  int nsplit;
  int cluster;
  int max_ctas;            // CTA budget of the call (0 = every SM)
  // query groups: G consecutive queries of one sequence share a work unit
  // (their G x n_h head rows form the MMA's 64 rows); n_qg = ceil(n_q / G)
  // groups per sequence.  G > 1 only for the all-entries (HCA) set with a
  // token-indexed window and one split per group.
  int G, n_qg;
  FastDiv fd_m, fd_nsplit, fd_nqg;   // divisions by m, nsplit and n_qg (set at launch)
  float *part_o;           // [B*n_q, nsplit, 64, c]
  float *part_ml;          // [B*n_q, nsplit, 64, 2]
};
size_t attend_workspace_bytes(const AttendParams &p);
int run_attend(const AttendParams &p, void *ws, size_t ws_bytes, cudaStream_t s);

// ------------------------------------------------------------- GEMM / glue
// C[M, N] = A[M, K] * B[N, K]^T (row-major, lda/ldb/ldc in elements).
int launch_gemm(hca_dtype ab_dtype, const void *A, long long lda, const void *Bm, long long ldb,
                void *C, long long ldc, hca_dtype c_dtype, int M, int N, int K, float alpha,
                cudaStream_t s);
// tcgen05 path of launch_gemm for bf16 A/B (M >= 128, N >= 256, K >= 64, 16-byte
// aligned rows); HCA_ERR_UNSUPPORTED (nothing launched) otherwise.
int launch_gemm_tc(const void *A, long long lda, const void *Bm, long long ldb, void *C, long long ldc,
                   hca_dtype c_dtype, int M, int N, int K, float alpha, cudaStream_t s);
// Row RMSNorm (optional) + partial RoPE (optional) + convert.  Row r of
// `rows` rows of `cols` values; the RoPE position is (pos0 + r / rows_per_pos) % pos_mod.
struct RowOpParams {
  const float *in; long long in_stride;
  void *out; long long out_stride; hca_dtype out_dtype;
  int rows, cols;
  int norm; const float *gamma; float eps;
  int rd; float theta; long long pos0; int rows_per_pos; int pos_mod;
  long long pos_base;   // RoPE position = pos_base + (pos0 + row / rows_per_pos) % pos_mod
  float scale;
  double rope_freq[32];  // filled by launch_row_op
};
int launch_row_op(const RowOpParams &p, cudaStream_t s);

}  // namespace hca
