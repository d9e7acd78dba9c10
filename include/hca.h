/*
 * hca.h -- C ABI of libhca, a B200 (sm_100a) implementation of DeepSeek-V4's
 * hybrid compressed attention: CSA (overlapped block compression, lightning
 * indexer + per-query top-k, shared-KV MQA) and HCA (heavy compression, dense
 * shared-KV MQA), both with a sliding-window branch, partial RoPE and a
 * per-head attention sink.
 *
 * Sources of the operations (page title, section / equation):
 *   [J] juejin "DeepSeek-V4 技术报告简要解读": §2.3.1 Eq.(9)-(19) (CSA),
 *       §2.3.2 Eq.(20)-(23) (HCA), §2.3.3 (QK norm, partial RoPE, window,
 *       sink Eq.(27)), §2.3.4 (mixed-precision KV storage), §4.4 (FP4
 *       indexer path, deferred), §4.6 (heterogeneous KV cache).
 *   [Z] 1zeryu "DeepSeek-V4：算法架构": "Q, K, V 映射与位置编码注入",
 *       "Sparse Attention", "CSA 选择器层代码实现" (Compressor, Indexer),
 *       "HCA 选择函数代码实现", "输出投影".
 *
 * Conventions (all functions):
 *   - Return HCA_OK (0) or a negative status; hca_last_error() gives text.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call launches nothing and changes no buffer.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous.  Nothing here synchronises except
 *     hca_check_status() and the diagnostics (hca_profile_sample,
 *     hca_trace_attend with counters).
 *   - Stream order is kept: a library kernel may be scheduled while the
 *     library kernel before it finishes (programmatic dependent launch), but
 *     it waits for that kernel's completion before touching any buffer.
 *   - The caller owns every device buffer.  The library allocates no device
 *     memory: scratch is passed as `ws` of at least the size the matching
 *     *_workspace_size() returns (256-byte aligned).
 *   - Tensors are dense, C-order, innermost dimension contiguous, base
 *     pointers 16-byte aligned.  Sizes below are in elements.
 *   - Index lists are int32; -1 marks an empty slot.
 *   - Positions are absolute token positions; one start position per call,
 *     shared by the whole batch.
 *   - Device-side waits are bounded; one that expires sets the device status
 *     word to HCA_ERR_TIMEOUT, the kernel returns, and hca_check_status()
 *     reports it.
 */
#ifndef HCA_H
#define HCA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *hca_stream_t; /* cudaStream_t */

enum {
  HCA_OK = 0,
  HCA_ERR_INVALID = -1,     /* bad shape, null / misaligned pointer, bad dtype */
  HCA_ERR_UNSUPPORTED = -2, /* valid request the library does not implement */
  HCA_ERR_CUDA = -3,        /* a CUDA runtime call failed (launch, attribute) */
  HCA_ERR_TIMEOUT = -4      /* a bounded device wait expired */
};

/* HCA_FP4: the FP4 indexer path ([J] §4.4; [Z] Indexer) -- indexer keys that
 * are Hadamard-rotated and FP4-quantised (E2M1, one power-of-two scale per 32
 * values, see hca_fp4_rotate_quant), carried exactly as bf16 values.  As an
 * idx_key_dtype it also rotates and quantises q^I inside csa_index_topk and
 * rounds the index scores to bf16 before the selection; as a compressor
 * out_dtype (width 64) the entries are rotated and quantised when written. */
typedef enum { HCA_F32 = 0, HCA_BF16 = 1, HCA_FP8E4M3 = 2, HCA_FP4 = 3 } hca_dtype;

/* ------------------------------------------------------------------------
 * Attention-layer shape.  Query i of a call sits at position start_pos + i.
 * Compressed entry s covers tokens [s*m, (s+1)*m) and is visible to query t
 * iff (s+1)*m <= t+1 ([Z] Indexer mask, get_compress_topk_idxs).
 * ---------------------------------------------------------------------- */
typedef struct {
  int B;                   /* sequences in the batch */
  int n_h;                 /* query heads sharing one KV head ([J] Eq.(18)) */
  int c;                   /* shared KV / head dim */
  int rd;                  /* RoPE dims: the last rd of c ([J] §2.3.3) */
  int w;                   /* sliding-window tokens, >= 0 */
  int m;                   /* compression ratio m (CSA) or m' (HCA) */
  int overlap;             /* 1: overlapped compression [J] Eq.(11)-(12) */
  int k;                   /* top-k entries per query (CSA) */
  int n_hI, c_I, rd_I;     /* indexer heads, head dim, RoPE dims ([J] Eq.(14)) */
  hca_dtype dtype;         /* storage of q, KV rows and o: HCA_F32 or HCA_BF16 */
  hca_dtype idx_key_dtype; /* indexer key cache: dtype or HCA_FP8E4M3 */
  float scale;             /* logit scale; <= 0 selects c^-1/2 */
  float eps;               /* RMSNorm epsilon (1e-6) */
  float rope_theta;        /* RoPE base (10000) */
  int max_ctas;            /* attention only: at most this many CTAs (one per SM) per
                              call, which also bounds the split-KV count per query;
                              0 = every SM.  For a caller that runs another layer's
                              kernels on a second stream at the same time. */
  int kv_mixed;            /* 1: the compressed KV rows and the window rows the layer
                              keeps are mixed-precision records (hca_kv_quant_mixed;
                              [J] §2.3.4): csa_attend / hca_attend read kv_comp and
                              kv_win as records of hca_kv_mixed_row_bytes(c, rd)
                              bytes and dequantise them on load (dtype HCA_BF16,
                              n_h <= 64, c in {128, 256, 512}).  0: dtype rows. */
} hca_attn_desc;

/* ------------------------------------------------------------------------
 * Block compression, [J] Eq.(11)-(12) (overlap = 1) or Eq.(22)-(23)
 * (overlap = 0); [Z] Compressor (prefill and decode branches).
 *
 * Entry i, channel ch: softmax over the rows of block i (logit Z_a + B_a) and,
 * with overlap and i > 0, the rows of block i-1 (logit Z_b + B_b); the entry
 * is the softmax-weighted sum of the matching C_a / C_b values.  With
 * HCA_COMPRESS_NORM the entry is then RMS-normalised (weight gamma, NULL =
 * ones); with HCA_COMPRESS_ROPE its last rd dims are rotated at position i*m.
 * ---------------------------------------------------------------------- */
#define HCA_COMPRESS_NORM 1
#define HCA_COMPRESS_ROPE 2

typedef struct {
  int B;               /* sequences */
  int width;           /* channels per entry (c, or c_I for indexer keys) */
  int m;               /* ratio */
  int overlap;         /* 1 = CSA overlapped series a/b, 0 = single series */
  int rd;              /* RoPE dims of the epilogue (<= width, even) */
  int flags;           /* HCA_COMPRESS_NORM | HCA_COMPRESS_ROPE */
  float eps, rope_theta;
  hca_dtype in_dtype;  /* C and Z rows: HCA_F32 or HCA_BF16 */
  hca_dtype out_dtype; /* entries: HCA_F32, HCA_BF16, HCA_FP8E4M3 or HCA_FP4 (width 64) */
} hca_compress_desc;

/* csa_compress -- two modes:
 *   prefill (start_pos == 0, n >= 1): writes entries 0 .. n/m - 1 of every
 *     sequence, and (if state_kv != NULL) leaves the compressor state ready
 *     for decode at position n.
 *   decode (start_pos > 0, n == 1): appends token start_pos to the state;
 *     when (start_pos + 1) % m == 0 writes entry start_pos / m.
 * Ca, Za [B, n, width] (row stride row_stride, sequence stride seq_stride,
 *   in elements); Cb, Zb the overlap series (NULL when overlap == 0).
 * Ba, Bb [m, width] fp32 position biases (Bb NULL when overlap == 0).
 * out: entry e of sequence b at out + (b*out_seq_stride + e)*width.
 * out_scale: fp32 [B, out_seq_stride] row scales, only for fp8 output.
 * state_kv / state_score fp32 [B, R, 2*width] (overlap, R = 2m) or
 *   [B, R, width] (R = m); rows 0..m-1 hold the previous block and rows
 *   m..2m-1 the current block (overlap); columns 0..width-1 the b series,
 *   width..2width-1 the a series; score rows carry the bias (Z + B); empty
 *   rows are (0, -inf).  Required in decode mode, optional in prefill. */
int csa_compress(const hca_compress_desc *d, int start_pos, int n,
                 const void *Ca, const void *Cb, const void *Za, const void *Zb,
                 long long row_stride, long long seq_stride,
                 const float *Ba, const float *Bb, const float *gamma,
                 void *out, float *out_scale, long long out_seq_stride,
                 float *state_kv, float *state_score, hca_stream_t stream);
/* hca_compress -- the same call under the HCA name (overlap = 0, ratio m'):
 * [J] Eq.(22)-(23); identical arguments and behaviour to csa_compress. */
int hca_compress(const hca_compress_desc *d, int start_pos, int n,
                 const void *Ca, const void *Cb, const void *Za, const void *Zb,
                 long long row_stride, long long seq_stride,
                 const float *Ba, const float *Bb, const float *gamma,
                 void *out, float *out_scale, long long out_seq_stride,
                 float *state_kv, float *state_score, hca_stream_t stream);

/* ------------------------------------------------------------------------
 * Lightning indexer score + per-query top-k, [J] Eq.(16)-(17); [Z] Indexer.
 *   I[t,s] = sum_h wI[t,h] * ReLU(qI[t,h] . K_I[s]) over visible s, then the
 *   min(k, V_t) highest scores (ties to the lower index), V_t = (t+1)/m.
 * qI [B, n_q, n_hI, c_I] (dtype; RoPE already applied), wI [B, n_q, n_hI]
 *   fp32 (already scaled), KI [B, cap, c_I] (idx_key_dtype), KI_scale
 *   [B, cap] fp32 row scales for fp8 keys (else NULL).
 * idx [B, n_q, k]: kept entry indices in ascending order, then -1.
 * idx_key_dtype HCA_FP4 (c_I = 64): KI holds rotated FP4 keys (bf16 storage,
 *   as csa_compress writes them); q^I is rotated and FP4-quantised in ws, the
 *   scores are rounded to bf16 (nearest, ties to even) before the selection
 *   (ties still to the lower index) and in the optional scores output.
 * scores (optional, NULL to skip): fp32 [B, n_q, score_stride] with the
 *   index scores of the visible entries (score_stride >= max V_t).
 * Requires (start_pos + n_q) / m <= cap. */
size_t csa_index_topk_workspace_size(const hca_attn_desc *d, int n_q, int start_pos);
int csa_index_topk(const hca_attn_desc *d, const void *qI, const float *wI,
                   const void *KI, const float *KI_scale, int cap, int n_q,
                   int start_pos, int32_t *idx, float *scores, long long score_stride,
                   void *ws, size_t ws_bytes, hca_stream_t stream);

/* The papers have no counterpart to this call: it is csa_index_topk (same
 * arguments, same results) for callers that cannot allocate or hand in a
 * workspace, e.g. an allocator's own out-of-memory path or a loop that must
 * not call cudaMalloc/cudaFree (they synchronise the device).  Its scratch is
 * a fixed device array of HCA_STATIC_SCRATCH_BYTES (8 MiB) per device, inside
 * the library; it allocates nothing.
 *   Needs csa_index_topk_workspace_size(d, n_q, start_pos) <=
 *   HCA_STATIC_SCRATCH_BYTES (about B*n_q*((start_pos+n_q)/m)*4 bytes, e.g. a
 *   decode step of 32 sequences at 131072 tokens with m = 4); a larger call
 *   fails with HCA_ERR_INVALID and a message naming both sizes.
 *   The first call on each device looks up the array's device address (with
 *   that device current); make it before any stream capture that includes
 *   this call.  The array is not cleared between calls and needs no clearing.
 *   The array is shared by every call on a device: calls that may overlap in
 *   time (different streams or host threads without ordering between them)
 *   race on it and must be serialised by the caller. */
#define HCA_STATIC_SCRATCH_BYTES (8u << 20)
/* HCA_STATIC_SCRATCH_BYTES as this build of the library has it (for callers
 * that load the library without its header, e.g. through ctypes). */
size_t hca_static_scratch_bytes(void);
int csa_index_topk_static_scratch(const hca_attn_desc *d, const void *qI, const float *wI,
                                  const void *KI, const float *KI_scale, int cap, int n_q,
                                  int start_pos, int32_t *idx, float *scores, long long score_stride,
                                  hca_stream_t stream);

/* ------------------------------------------------------------------------
 * Shared-KV MQA with sink, [J] Eq.(18)-(19), (27), §2.3.3; [Z] Sparse
 * Attention, 输出投影.  For query t (head h) the key/value rows are the
 * window rows of tokens max(0, t-w+1) .. t followed by the compressed rows
 * (csa_attend: idx[t, j] >= 0; hca_attend: every visible entry s < (t+1)/m).
 *   z_j = scale * q_h . row_j ; o_h = sum_j e^{z_j} row_j / (sum_j e^{z_j} + e^{sink_h})
 * then the last rd dims of o_h are rotated by -t.
 * q [B, n_q, n_h, c]; kv_comp [B, cap, c]; sink [n_h] fp32; o [B, n_q, n_h, c].
 * kv_win: token rows (win_is_ring == 0): [B, h + n_q, c], row r = token
 *   start_pos - h + r, where h = min(w - 1, start_pos) is the halo of window
 *   rows before the first query (h = 0 for a prefill from position 0; a
 *   context-parallel rank starting at start_pos > 0 passes its halo);
 *   decode (win_is_ring == 1, n_q == 1): [B, w, c] ring, token p in slot
 *   p % w (the caller has already stored token start_pos).
 * Few queries (decode): each query's key list is cut across up to 8 CTAs of a
 *   thread-block cluster whose partials are merged on chip; no scratch needed.
 * ws: scratch only for a query cut into more than 8 pieces (fp32 partials +
 *   a merge launch); *_attend_workspace_size() gives its size (0 when not
 *   needed).  With ws == NULL or too small such a call is cut into 8 pieces
 *   instead (same result up to fp32 rounding order). */
size_t csa_attend_workspace_size(const hca_attn_desc *d, int n_q, int start_pos);
int csa_attend(const hca_attn_desc *d, const void *q, const void *kv_comp, int cap,
               const int32_t *idx, const void *kv_win, int win_is_ring,
               const float *sink, int n_q, int start_pos, void *o,
               void *ws, size_t ws_bytes, hca_stream_t stream);

size_t hca_attend_workspace_size(const hca_attn_desc *d, int n_q, int start_pos);
int hca_attend(const hca_attn_desc *d, const void *q, const void *kv_comp, int cap,
               const void *kv_win, int win_is_ring, const float *sink, int n_q,
               int start_pos, void *o, void *ws, size_t ws_bytes, hca_stream_t stream);

/* ------------------------------------------------------------------------
 * Whole layer.  Weights are stored [d_out, d_in] row-major in a.dtype.
 * ---------------------------------------------------------------------- */
typedef enum { HCA_LAYER_CSA = 0, HCA_LAYER_HCA = 1, HCA_LAYER_SWA = 2 } hca_layer_kind;

typedef struct {
  hca_layer_kind kind;
  hca_attn_desc a;
  int d;               /* d_model */
  int d_c;             /* query compression rank ([J] Eq.(13)) */
  const void *W_comp;  /* CSA [4c, d] = W_aKV|W_bKV|W_aZ|W_bZ; HCA [2c, d] = W_KV|W_Z */
  const float *B_comp; /* CSA [2, m, c] = B_a, B_b; HCA [m, c] */
  const void *W_compI; /* CSA indexer compressor [4c_I, d] */
  const float *B_compI;/* CSA [2, m, c_I] */
  const void *W_DQ;    /* [d_c, d]        c^Q = RMSNorm(h W_DQ)          */
  const void *W_UQ;    /* [n_h*c, d_c]    q = c^Q W_UQ, per-head RMS, RoPE */
  const void *W_IUQ;   /* [n_hI*c_I, d_c] q^I = c^Q W_IUQ, RoPE (CSA)     */
  const void *W_w;     /* [n_hI, d]       w^I = h W_w * c_I^-1/2 n_hI^-1/2 */
  const void *W_KV;    /* [c, d]          window kv = RMSNorm(h W_KV), RoPE */
  const float *sink;   /* [n_h] */
} hca_layer;

/* Decode-time cache of one layer ([J] §4.6: fixed-size state + classical
 * compressed cache).  All device memory, owned by the caller. */
typedef struct {
  int cap;             /* entries per sequence (multiple of lcm(m, m')/m) */
  void *kv_comp;       /* [B, cap, c] a.dtype */
  void *key_I;         /* [B, cap, c_I] idx_key_dtype (CSA) */
  float *key_I_scale;  /* [B, cap] (fp8 keys) */
  void *win;           /* [B, w, c] ring, token p in slot p % w */
  float *state_kv, *state_score;   /* compressor state (see csa_compress) */
  float *stateI_kv, *stateI_score; /* indexer compressor state (CSA) */
} hca_cache;

/* hybrid_layer_forward -- prefill of n tokens per sequence from hidden states
 * H [B, n, d] (a.dtype) at positions 0 .. n-1; writes o [B, n, n_h, c].
 * With cache != NULL also fills the compressed caches, the window ring and
 * the compressor states so that decode can continue at position n. */
size_t hybrid_layer_forward_workspace_size(const hca_layer *L, int n);
int hybrid_layer_forward(const hca_layer *L, const void *H, int n, hca_cache *cache,
                         void *o, void *ws, size_t ws_bytes, hca_stream_t stream);

/* One decode token per sequence: the projected inputs of the new token. */
typedef struct {
  const void *q;       /* [B, n_h, c] normalised, RoPE'd at pos */
  const void *qI;      /* [B, n_hI, c_I] RoPE'd at pos (CSA) */
  const float *wI;     /* [B, n_hI] scaled (CSA) */
  const void *kv;      /* [B, c] window row (normalised, RoPE'd at pos) */
  const float *comp;   /* [B, 4c] (CSA: Ca|Cb|Za|Zb) or [B, 2c] (HCA: C|Z) fp32 */
  const float *compI;  /* [B, 4c_I] (CSA) fp32 */
} hca_token_in;

/* hybrid_decode_inputs -- the decode token's inputs from hidden states:
 * h [B, d] (a.dtype) holds one token per sequence, all at position pos; the
 * call writes the buffers that x points to (allocated by the caller with the
 * sizes above; the const qualifiers are for hybrid_decode_step, which reads
 * them): comp = h W_comp^T (fp32, [J] Eq.(9)-(10) / (20)-(21)); q = per-head
 * RMSNorm of RMSNorm(h W_DQ^T) W_UQ^T, RoPE'd at pos (Eq.(13), (18)); kv =
 * RMSNorm(h W_KV^T) RoPE'd at pos (the window row, when w > 0); for CSA also
 * compI = h W_compI^T, qI = RoPE(RMSNorm(h W_DQ^T) W_IUQ^T) at pos (Eq.(14)),
 * wI = h W_w^T c_I^-1/2 n_hI^-1/2 (Eq.(15)).  These are the prefill's
 * projections restricted to one token, so a layer's output, projected to
 * hidden states (hca_output_projection and the caller's residual path), can
 * feed the next layer's decode step.  Workspace: fp32 / bf16 intermediates
 * (hybrid_decode_inputs_workspace_size).  Errors: HCA_ERR_INVALID for a null h
 * or x, a missing output buffer, pos < 0 or a short workspace. */
size_t hybrid_decode_inputs_workspace_size(const hca_layer *L);
int hybrid_decode_inputs(const hca_layer *L, const void *h, int pos, const hca_token_in *x, void *ws,
                         size_t ws_bytes, hca_stream_t stream);

/* hybrid_decode_step -- token at position pos (> 0) for every sequence:
 * stores its window row, advances the compressor states (emitting an entry
 * when (pos+1) % m == 0), scores and selects (CSA), and attends; writes
 * o [B, n_h, c]. */
size_t hybrid_decode_step_workspace_size(const hca_layer *L, int pos);
int hybrid_decode_step(const hca_layer *L, const hca_token_in *x, hca_cache *cache,
                       int pos, void *o, void *ws, size_t ws_bytes, hca_stream_t stream);

/* ------------------------------------------------------------------------
 * Context-parallel prefill ([J] §4.5, the two-stage communication for
 * compressed attention; ranhao §6): the tokens of a long prefill are cut into
 * contiguous ranges, one per rank.  Stage 1 compresses each range on its own
 * (hybrid_cp_compress); the caller then all-gathers the ranks' entries and
 * indexer keys (one collective, e.g. NCCL); stage 2 scores, selects and
 * attends the range's queries against the gathered caches (hybrid_cp_attend).
 * A rank owns tokens [t0, t0 + n_loc) of every sequence (t0 a multiple of m)
 * and is given H [B, h + n_loc, d] (a.dtype): its rows preceded by the
 * h = hybrid_cp_halo(L, t0) rows of the tokens before t0 (the window rows of
 * its first queries, and for CSA the previous block, whose b series the
 * range's first entry needs).  Compressed layers only (CSA, HCA); a CSA
 * window must cover the overlap block (w - 1 >= m).
 * ---------------------------------------------------------------------- */
/* h = min(t0, max(w - 1, m if the layer's compression overlaps else 0)). */
int hybrid_cp_halo(const hca_layer *L, int t0);
size_t hybrid_cp_workspace_size(const hca_layer *L, int t0, int n_loc);
/* Stage 1: entries t0/m .. (t0 + n_loc)/m - 1 of every sequence, normalised
 * and RoPE'd at their global positions, to kv_comp [B, out_cap, c] (a.dtype)
 * and, CSA, key_I [B, out_cap, c_I] (idx_key_dtype; key_I_scale [B, out_cap]
 * fp32 for fp8 keys), slots 0 .. n_loc/m - 1. */
int hybrid_cp_compress(const hca_layer *L, const void *H, int t0, int n_loc, void *kv_comp, void *key_I,
                       float *key_I_scale, int out_cap, void *ws, size_t ws_bytes, hca_stream_t stream);
/* Stage 2: o [B, n_loc, n_h, c] of the range's queries against the gathered
 * caches kv_comp [B, cap, c] and (CSA) key_I [B, cap, c_I] (+ key_I_scale),
 * which must hold entries 0 .. (t0 + n_loc)/m - 1 (cap >= that). */
int hybrid_cp_attend(const hca_layer *L, const void *H, int t0, int n_loc, const void *kv_comp, const void *key_I,
                     const float *key_I_scale, int cap, void *o, void *ws, size_t ws_bytes, hca_stream_t stream);

/* Where the two calls above leave their intermediate results inside the
 * caller's workspace, so that a caller can inspect the selection and the
 * stored operands after the call (they stay until the workspace is reused).
 * decode = 0 describes hybrid_layer_forward(L, ., n, ...), decode = 1
 * hybrid_decode_step(L, ., ., pos = n, ...).  Each field is a byte offset
 * from ws, or -1 when the call has no such buffer (another layer kind, decode,
 * or a prefill with a cache, which stores entries and keys in the cache):
 *   idx     [B, n_q, k] int32   kept entries (CSA), ascending, -1 padded
 *   q       [B, n, n_h, c]      queries, normalised and RoPE'd   (a.dtype)
 *   qI      [B, n, n_hI, c_I]   index queries, RoPE'd           (a.dtype)
 *   wI      [B, n, n_hI] fp32   index weights (scaled)
 *   key_I   [B, n/m, c_I]       indexer keys                     (a.dtype)
 *   kv_comp [B, n/m, c]         compressed entries               (a.dtype)
 *   kv_win  [B, n, c]           window rows, normalised, RoPE'd  (a.dtype)
 * (n_q = n for prefill, 1 for decode.)  Returns HCA_ERR_INVALID for a bad
 * layer, n < 0 (prefill) or n < 1 (decode). */
typedef struct {
  long long idx, q, qI, wI, key_I, kv_comp, kv_win;
} hca_ws_map;
int hybrid_workspace_map(const hca_layer *L, int n, int decode, hca_ws_map *map);

/* ------------------------------------------------------------------------
 * Grouped output projection, [J] §2.3.1(d); [Z] 输出投影 -- the step after the
 * attention.  o [T, n_h, c] (inverse RoPE already applied, dtype) is split into
 * g groups of n_h/g consecutive heads; group i's n_h*c/g values go through
 * wo_a[i] to d_g values:  mid_i = o_i . wo_a[i]^T  (wo_a [g, d_g, n_h*c/g]);
 * out [T, d] = concat_i(mid_i) . wo_b^T  (wo_b [d, g*d_g]).  Weights are
 * row-major in dtype (f32 or bf16); out is f32 or bf16 (out_dtype).  The
 * intermediate [T, g*d_g] is kept in ws in dtype (bf16 rounding for bf16).
 * Requires n_h % g == 0; pointers 16-byte aligned. */
typedef struct {
  int T, n_h, c, g, d_g, d;
  hca_dtype dtype, out_dtype;
} hca_oproj_desc;
size_t hca_output_projection_workspace_size(const hca_oproj_desc *d);
int hca_output_projection(const hca_oproj_desc *d, const void *o, const void *wo_a, const void *wo_b,
                          void *out, void *ws, size_t ws_bytes, hca_stream_t stream);

/* ------------------------------------------------------------------------
 * Status and diagnostics.
 * ---------------------------------------------------------------------- */
const char *hca_last_error(void);   /* text of the last failing call (thread-local) */
/* Synchronises `stream`, then reads and clears the device status word that
 * kernels set when a bounded wait expires.  *device_status = HCA_OK or
 * HCA_ERR_TIMEOUT.  Returns HCA_ERR_CUDA if the synchronisation failed. */
int hca_check_status(hca_stream_t stream, int *device_status);
/* Failure-detection self-test (no counterpart in the papers): launches one
 * block whose single mbarrier wait can never complete.  The wait gives up
 * after limit_ns (1 ms .. 2 s), sets the status word to HCA_ERR_TIMEOUT and
 * the kernel returns, exactly as an expired wait in the production kernels
 * does; the CUDA context stays usable.  Returns HCA_ERR_INVALID for a limit
 * out of range, else the launch status. */
int hca_selftest_wait(unsigned long long limit_ns, hca_stream_t stream);
int hca_version(void);              /* (major << 16) | minor */
/* Kernels launched by the library since load (per process), for accounting. */
long long hca_launch_count(void);
/* Per-kernel timing: with profiling on, every launch is bracketed by CUDA
 * events recorded on its own stream (also inside a CUDA graph capture, where
 * the records become graph nodes).  hca_profile_sample() waits for the
 * recorded events and adds their durations to per-kernel counters, keeping
 * the records (call it after each replay of a captured graph, or after each
 * step).  hca_profile_collect() writes one line per kernel name
 * "name<TAB>launches<TAB>total_ms\n" into buf (NUL-terminated), then clears
 * the counters and the records.  Returns HCA_ERR_INVALID if buf is too small. */
int hca_profile_enable(int on);
int hca_profile_sample(void);
int hca_profile_collect(char *buf, size_t len);
/* ------------------------------------------------------------------------
 * Mixed-precision KV rows, [J] §2.3.4 (the KV cache keeps the RoPE dims in
 * BF16 and the other dims in FP8, nearly halving it); [Z] "Q, K, V 映射与位置
 * 编码注入" and Compressor (after RoPE, the non-RoPE dims of each KV row are
 * quantised to FP8 in blocks of 64 channels).
 *
 * Record of one row, hca_kv_mixed_row_bytes(c, rd) bytes (a multiple of 16):
 *   bytes [0, c-rd)                 e4m3 codes of channels 0 .. c-rd-1
 *   bytes [c-rd, c+rd)              channels c-rd .. c-1 (the RoPE dims) as bf16
 *   bytes [c+rd, c+rd+(c-rd)/16)    one fp32 scale per 64 code channels
 *   then zero bytes up to the record size (c = 512, rd = 64: 604 -> 608 bytes).
 * Block scale = block amax / 448 and code = nearest e4m3 (ties to even,
 * saturating) of x / scale, both divisions rounded to fp32; zero is stored
 * as +0 and an all-zero block gets scale 0.  Shapes: c <= 512, rd a multiple
 * of 16, c - rd a multiple of 64.  Inputs must be finite.
 * ---------------------------------------------------------------------- */
/* Record bytes of one row; 0 when (c, rd) is unsupported. */
size_t hca_kv_mixed_row_bytes(int c, int rd);
/* x: [rows, c] HCA_F32 or HCA_BF16 rows (row stride c, 16-byte aligned);
 * out: rows consecutive records (16-byte aligned, caller-owned).  rows = 0
 * is a no-op.  HCA_ERR_INVALID for a bad shape, dtype or pointer. */
int hca_kv_quant_mixed(const void *x, hca_dtype x_dtype, long long rows, int c, int rd, void *out,
                       hca_stream_t stream);
/* in: rows records; out: [rows, c] bf16 rows, each code channel
 * bf16(fp32(code * scale)) (nearest, ties to even), the RoPE channels copied. */
int hca_kv_dequant_mixed(const void *in, long long rows, int c, int rd, void *out, hca_stream_t stream);

/* ------------------------------------------------------------------------
 * FP4 indexer activations, [J] §4.4 (the indexer's QK activations in FP4 E2M1
 * with scales per 1 x 32 sub-block that FP8 absorbs losslessly, i.e. powers of
 * two); [Z] Indexer (q^I and the keys Hadamard-rotated first).
 *
 * x: [rows, n] HCA_F32 or HCA_BF16 (n = 64); out: [rows, n] bf16.  Each row is
 * rotated by the orthonormal Hadamard matrix (butterflies of strides 1, 2, ...
 * in fp32, then the exact scale n^-1/2), cut into blocks of 32 with scale
 * 2^(floor(log2 amax) - 2), rounded to E2M1 (nearest, ties to even, saturating
 * at 6; zero as +0) and written as bf16 -- exact, since every E2M1 value times
 * a power of two is a bf16 value.  rows = 0 is a no-op.
 * ---------------------------------------------------------------------- */
int hca_fp4_rotate_quant(const void *x, hca_dtype x_dtype, long long rows, int n, void *out, hca_stream_t stream);

/* Diagnostic timeline of the decode step's kernels (ingest, indexer, top-k,
 * attention): with buf set, thread 0 of every CTA of those kernels appends
 * one record of four uint64 -- entry time, time after its wait for the
 * previous kernel, exit time (all %globaltimer ns) and kernel << 48 | SM << 32
 * | CTA index (kernel: 1 ingest, 2 indexer, 3 top-k, 4 CSA attention, 5 HCA
 * attention) -- at buf + 8 + 32 * i, where i comes from the uint64 counter at
 * buf[0] (records past the capacity are counted, not written).  The caller
 * zeroes buf and reads it after synchronising.  buf = NULL switches it off.
 * Synchronises the device (it sets a device variable per source file). */
int hca_step_trace(void *buf, size_t bytes);

/* Diagnostic trace of the tensor-core attention kernel: with enable = 1 the
 * following attend launches accumulate, summed over CTAs, the SM cycles each
 * role spends waiting on each pipeline barrier, plus unit / tile / rescale
 * counts (slot order: producer Q-free, producer stage-free, MMA Q-ready, MMA
 * tile-ready, MMA S-free, MMA P-ready, MMA O-free, softmax S-ready, softmax
 * P-buffer-free, softmax rescale wait, softmax epilogue wait, -, epilogue
 * cycles, total cycles, rescales, units, tiles).  host_counters (n slots,
 * may be NULL) receives the counters (the call synchronises the device);
 * enable >= 0 then resets them and sets the mode, enable < 0 only reads. */
int hca_trace_attend(int enable, unsigned long long *host_counters, int n);

/* Which kernel runs the top-k selection of csa_index_topk (and of the layer
 * calls that use it), for tests and measurements: 0 = chosen by shape (the
 * default), 1 = one CTA per row (rows of up to 32768 keys in registers),
 * 2 = one warp per row (rows of up to 32768 keys; many rows), 3 = the
 * segmented cluster radix select, 4 = one thread-block cluster per row
 * (rows all longer than k).  A mode whose kernel does not take the shape
 * falls back to the segmented select, so every mode is exact for every
 * shape.  Returns the previous mode;
 * mode < 0 only reads it.  Process-wide setting (not per device or stream);
 * workspace sizes depend on it for mode 3, so size workspaces after setting
 * it.  Errors: HCA_ERR_INVALID for mode > 4. */
int hca_topk_kernel(int mode);

#ifdef __cplusplus
}
#endif

#endif /* HCA_H */
