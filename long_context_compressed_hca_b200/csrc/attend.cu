// attend.cu -- shared-KV MQA with a sliding-window branch and attention sink.
//
// For query token t and head h (juejin "DeepSeek-V4 技术报告简要解读" §2.3.1(c)
// Eq.(18)-(19), §2.3.3 Eq.(27); 1zeryu "DeepSeek-V4：算法架构", Sparse
// Attention / 输出投影):
//   rows  = window rows of tokens max(0,t-w+1)..t, then the compressed rows
//           (CSA: idx[t, j] for the first min(k, V_t) slots; HCA: entries 0..V_t-1)
//   z_j   = scale * q_h . row_j
//   o_h   = sum_j e^{z_j} row_j / (sum_j e^{z_j} + e^{sink_h})
//   o_h[last rd dims] rotated by -t.
// Every row is both key and value; all n_h heads share it.
//
// Two implementations:
//   attend_tc   bf16, tcgen05.  One query token per work unit, its n_h (<= 64)
//               heads form the M=64 rows.  Q sits in tensor memory (written by
//               the softmax warps) and is the A operand of S = Q K^T, which
//               lands per 64-key tile in a TMEM accumulator in lane-half 1
//               (double buffered); softmax in registers, P (bf16) to shared
//               memory, O += P V into a TMEM accumulator in lane-half 0 (up to
//               512 fp32 columns).  The key tile in shared memory (3 stages at
//               c = 512) serves as K (K-major) and V (MN-major).  Warp roles:
//               4 softmax/epilogue warps, 1 MMA warp, 8 gather warps (cp.async
//               of the selected rows into 128B-swizzled tiles).  Few queries:
//               a query's tiles are split over the CTAs of a cluster and
//               merged in distributed shared memory.
//   attend_simt fp32 CUDA cores, any shape (and the tiny fp32 workload).
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

struct KeySet {
  int nw, nw4, nc, nk, t0, V;   // window keys, window slots (multiple of 4), compressed, total slots
};

__device__ __forceinline__ KeySet key_set(const AttendParams &p, int qi) {
  KeySet k;
  const int t = p.start_pos + qi;
  k.V = fdiv(t + 1, p.fd_m);
  k.nw = min(p.w, t + 1);
  k.t0 = t - k.nw + 1;
  k.nc = p.csa ? min(p.k, k.V) : k.V;
  k.nw4 = k.nw;
  k.nk = k.nw + k.nc;
  return k;
}

// Key slots of the tensor-core path: window keys in slots [0, nw), padding to
// a multiple of 4 (masked), compressed keys from slot nw4, so that every
// group of 4 slots comes from one tensor.
__device__ __forceinline__ KeySet key_set_tc(const AttendParams &p, int qi) {
  KeySet k = key_set(p, qi);
  k.nw4 = (k.nw + 3) & ~3;
  k.nk = k.nw4 + k.nc;
  return k;
}

// Work unit u: sequence b, query group qg (queries qi0 .. qi0 + G - 1), split sp.
struct Unit {
  int bq, b, qg, qi0, sp;
};
__device__ __forceinline__ Unit unit_of(const AttendParams &p, int u) {
  Unit x;
  x.bq = fdiv(u, p.fd_nsplit);
  x.sp = u - x.bq * p.nsplit;
  x.b = fdiv(x.bq, p.fd_nqg);
  x.qg = x.bq - x.b * p.n_qg;
  x.qi0 = x.qg * p.G;
  return x;
}

// Key slots of query group qg: the union of its queries' windows -- one run
// of tokens, from the first query's first window token to the last query --
// and the last query's visible entries (the most any query of the group
// sees).  Each query masks the slots outside its own key set.
__device__ __forceinline__ KeySet group_key_set(const AttendParams &p, int qg) {
  if (p.G == 1) return key_set_tc(p, qg);
  const int qi0 = qg * p.G;
  const int qi1 = min(p.n_q, qi0 + p.G) - 1;
  const KeySet a = key_set(p, qi0);
  KeySet k = key_set(p, qi1);
  k.t0 = a.t0;
  k.nw = p.w > 0 ? (p.start_pos + qi1) - a.t0 + 1 : 0;
  k.nw4 = (k.nw + 3) & ~3;
  k.nk = k.nw4 + k.nc;
  return k;
}

// Whether slot kk (< nk) of a group's key set is a key of query token tq:
// a window token in (tq - w, tq], or one of its (tq + 1) / m visible entries.
__device__ __forceinline__ bool slot_of_token(const AttendParams &p, const KeySet &ks, int kk, int tq) {
  if (kk < ks.nw4) {
    const int tok = ks.t0 + kk;
    return kk < ks.nw && tok <= tq && tok > tq - p.w;
  }
  return kk - ks.nw4 < fdiv(tq + 1, p.fd_m);
}

// Source row of slot kk (window tensor if kk < nw4, else compressed tensor)
// and whether it is a real key; masked slots point at a valid row.
__device__ __forceinline__ int slot_row(const AttendParams &p, const KeySet &ks, int b, int qi, int kk,
                                        bool &valid) {
  if (kk < ks.nw4) {
    valid = kk < ks.nw;
    const int tok = valid ? ks.t0 + kk : ks.t0 + ks.nw - 1;
    return p.win_is_ring ? b * p.w + tok % p.w : b * p.win_rows + (tok - p.win_tok0);
  }
  const int slot = kk - ks.nw4;
  int e = slot;
  valid = slot < ks.nc;
  if (valid && p.csa) {
    e = p.idx[((long long)b * p.n_q + qi) * p.k + slot];
    valid = e >= 0 && e < ks.V;
  }
  return b * p.cap + (valid ? e : 0);
}

// Row pointer of key `j` of query (b, qi), or nullptr if the slot is empty.
template <typename T>
__device__ __forceinline__ const T *key_row(const AttendParams &p, const KeySet &ks, int b, int qi,
                                            int j) {
  if (j < ks.nw) {
    const int tok = ks.t0 + j;
    if (p.win_is_ring)
      return reinterpret_cast<const T *>(p.kv_win) + ((long long)b * p.w + tok % p.w) * p.c;
    return reinterpret_cast<const T *>(p.kv_win) + ((long long)b * p.win_rows + (tok - p.win_tok0)) * p.c;
  }
  if (j >= ks.nk) return nullptr;
  int e = j - ks.nw;
  if (p.csa) {
    e = p.idx[((long long)b * p.n_q + qi) * p.k + e];
    if (e < 0 || e >= ks.V) return nullptr;
  }
  return reinterpret_cast<const T *>(p.kv_comp) + ((long long)b * p.cap + e) * p.c;
}

// Tile range [j0, j0 + nt) of split `sp` of a query's key list.
__device__ __forceinline__ void split_range(const KeySet &ks, int nsplit, int sp, int &j0, int &nt) {
  const int all = (ks.nk + 63) / 64;
  const int per = (all + nsplit - 1) / nsplit;
  j0 = sp * per;
  const int j1 = min(all, j0 + per);
  nt = j1 > j0 ? j1 - j0 : 0;
}

// Merge the split partials of one query: o_h = sum_s 2^{m_s-M} O_s /
// (sum_s 2^{m_s-M} l_s + 2^{sink_h-M}), then the inverse RoPE at t.
// Block = (query, group of 4 heads); thread = 4 consecutive columns.
template <typename T>
__global__ void __launch_bounds__(128) attend_combine(AttendParams p) {
  __shared__ float wsc[4][32];
  __shared__ float inv_den[4];
  __shared__ float rcs[64];          // cos[32], sin[32] of the token's RoPE pairs
  const int bq = blockIdx.x, hg = blockIdx.y;
  const int qi = bq % p.n_q, b = bq / p.n_q;
  const int t = p.start_pos + qi;
  const KeySet ks = key_set_tc(p, qi);
  const int C = p.c;
  if (threadIdx.x < 4) {
    const int r = hg * 4 + threadIdx.x;
    const float sink2 = p.sink[r < p.n_h ? r : 0] * kLog2e;
    float M = sink2;
    for (int sp = 0; sp < p.nsplit; ++sp) {
      int j0, nt;
      split_range(ks, p.nsplit, sp, j0, nt);
      if (nt) M = fmaxf(M, p.part_ml[(((long long)bq * p.nsplit + sp) * 64 + r) * 2]);
    }
    float den = exp2f(sink2 - M);
    for (int sp = 0; sp < p.nsplit; ++sp) {
      int j0, nt;
      split_range(ks, p.nsplit, sp, j0, nt);
      float w = 0.f;
      if (nt) {
        const float *ml = p.part_ml + (((long long)bq * p.nsplit + sp) * 64 + r) * 2;
        w = exp2f(ml[0] - M);
        den += w * ml[1];
      }
      wsc[threadIdx.x][sp] = w;
    }
    inv_den[threadIdx.x] = 1.f / den;
  } else if (threadIdx.x >= 32 && threadIdx.x - 32 < p.rd / 2) {
    const int i = threadIdx.x - 32;
    float sn, cs;
    rope_sincos_tab(p.rope_freq, t, i, p.rd, p.theta, &sn, &cs);
    rcs[i] = cs;
    rcs[32 + i] = sn;
  }
  __syncthreads();
  const int per_head = C / 4;
  for (int e = threadIdx.x; e < 4 * per_head; e += blockDim.x) {
    const int hh = e / per_head, r = hg * 4 + hh;
    const int col = 4 * (e % per_head);
    if (r >= p.n_h) continue;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float *base = p.part_o + ((long long)bq * p.nsplit * 64 + r) * C + col;
#pragma unroll 4
    for (int sp = 0; sp < p.nsplit; ++sp) {
      const float w = wsc[hh][sp];
      const float4 v = *reinterpret_cast<const float4 *>(base + (long long)sp * 64 * C);
      acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
    }
    const float id = inv_den[hh];
    float v[4] = {acc.x * id, acc.y * id, acc.z * id, acc.w * id};
    if (col + 4 > C - p.rd) {
#pragma unroll
      for (int x = 0; x < 4; x += 2) {
        if (col + x >= C - p.rd) {
          const int pi = (col + x - (C - p.rd)) / 2;
          const float cs = rcs[pi], sn = rcs[32 + pi];
          const float a = v[x], bb = v[x + 1];
          v[x] = a * cs + bb * sn;
          v[x + 1] = -a * sn + bb * cs;
        }
      }
    }
    T *orow = reinterpret_cast<T *>(p.o) + (((long long)b * p.n_q + qi) * p.n_h + r) * C + col;
#pragma unroll
    for (int x = 0; x < 4; ++x) Elt<T>::store(orow + x, v[x]);
  }
}

// ======================================================================= SIMT
constexpr int kSimtWarps = 8;
constexpr int kSimtKT = 16;

template <typename T>
__global__ void __launch_bounds__(kSimtWarps * 32) attend_simt(AttendParams p) {
  extern __shared__ float ks[];   // [kSimtKT][c]
  __shared__ int kvalid[kSimtKT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = blockIdx.x % p.n_q, b = blockIdx.x / p.n_q;
  const int h = blockIdx.y * kSimtWarps + warp;
  const bool hact = h < p.n_h;
  const int E = p.c / 32;
  const KeySet kset = key_set(p, qi);
  const float zs = p.scale * kLog2e;
  float qv[16], acc[16];
  const T *qrow = reinterpret_cast<const T *>(p.q) + (((long long)b * p.n_q + qi) * p.n_h + (hact ? h : 0)) * p.c;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    qv[i] = (i < E) ? Elt<T>::load(qrow + lane + 32 * i) * zs : 0.f;
    acc[i] = 0.f;
  }
  float mrun = -INFINITY, l = 0.f;
  for (int j0 = 0; j0 < kset.nk; j0 += kSimtKT) {
    for (int e = threadIdx.x; e < kSimtKT * p.c; e += blockDim.x) {
      const int r = e / p.c, col = e % p.c;
      const T *row = key_row<T>(p, kset, b, qi, j0 + r);
      ks[e] = row ? Elt<T>::load(row + col) : 0.f;
      if (col == 0) kvalid[r] = row != nullptr;
    }
    __syncthreads();
    const int nrow = min(kSimtKT, kset.nk - j0);
    for (int r = 0; r < nrow; ++r) {
      if (!kvalid[r]) continue;
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < E) part += qv[i] * ks[r * p.c + lane + 32 * i];
      const float z = warp_sum(part);
      const float mn = fmaxf(mrun, z);
      const float sc = exp2f(mrun - mn);
      const float pz = exp2f(z - mn);
      l = l * sc + pz;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < E) acc[i] = acc[i] * sc + pz * ks[r * p.c + lane + 32 * i];
      mrun = mn;
    }
    __syncthreads();
  }
  if (!hact) return;
  const float sink2 = p.sink[h] * kLog2e;
  const float M = fmaxf(mrun, sink2);
  const float sc = (mrun == -INFINITY) ? 0.f : exp2f(mrun - M);
  const float denom = l * sc + exp2f(sink2 - M);
  const float inv = sc / denom;
  const int t = p.start_pos + qi;
  T *orow = reinterpret_cast<T *>(p.o) + (((long long)b * p.n_q + qi) * p.n_h + h) * p.c;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (i >= E) continue;
    const int col = lane + 32 * i;
    float v = acc[i] * inv;
    const float other = __shfl_xor_sync(0xffffffffu, v, 1);
    if (col >= p.c - p.rd) {
      float s, cs;
      rope_sincos_tab(p.rope_freq, t, (col - (p.c - p.rd)) / 2, p.rd, p.theta, &s, &cs);
      // inverse rotation: (a, b) -> (a cos + b sin, -a sin + b cos)
      v = (lane & 1) ? (-other * s + v * cs) : (v * cs + other * s);
    }
    Elt<T>::store(orow + col, v);
  }
}

// CTAs one call may occupy: the caller's budget, else every SM.
inline int sm_budget(const AttendParams &p) {
  const int n = num_sms();
  return p.max_ctas > 0 && p.max_ctas < n ? p.max_ctas : n;
}

// ======================================================================= tcgen05
namespace tc {
bool g_trace_on = false;
bool attend_trace_on() { return g_trace_on; }
constexpr int KT = 64;
constexpr int kSoftmaxWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kProdWarp0 = 5;
constexpr int kProdWarps = 8;
constexpr int kProdThreads = kProdWarps * 32;
constexpr int kThreads = (kSoftmaxWarps + 1 + kProdWarps) * 32;
constexpr uint32_t kTileBytes = 64 * 128;   // 64 rows x 128 B (one 64-column block)
constexpr int kMaxClusterSplits = 8;         // portable cluster size
// S / P buffers and how many S tiles the MMA issue runs ahead of P.V.  Two
// tiles ahead measured slower than one (the third key stage then refills only
// after P.V(j-1) and the gathers stall the tensor pipe), so one: S(j+1) is
// queued behind P.V(j-1) while the softmax of tile j runs.
constexpr int kSP = 2;
constexpr int kLookahead = 1;

struct Bars {
  uint64_t q_full, q_empty, o_empty, mma_done;
  uint64_t kv_full[8], kv_empty[8], s_full[3], s_empty[3], p_full[3], pv_done[3];
  uint64_t mg_ready, mg_full;    // cluster merge: peers' buffers free / peers' partials delivered
  uint64_t mg_stage;             // cluster merge: this CTA's blocks staged
  uint64_t pair[4];              // M = 128: the two softmax warps of a TMEM lane quarter
  uint64_t us_full[2], us_empty[2];   // M = 128: unit slots (staged Q + RoPE table)
};

// Shared and tensor memory of one CTA.  M = 64: one query's (or a group's)
// heads on 64 rows, S and Q in TMEM lane-half 1 beside O in lane-half 0.
// M = 128 (c = 128, query groups): row i in TMEM lane i; two O accumulators
// (one per half of each key tile), S buffers, Q; the loaders stage each
// unit's Q rows and RoPE table in shared memory ahead of it.
template <int C, int M = 64>
struct Layout {
  static_assert(M == 64 || (M == 128 && C == 128), "M = 128 rows need c = 128");
  static constexpr int NKB = C / 64;
  // key-tile stages: Q lives in tensor memory, so the stages take what the P
  // buffers leave (192 KB for C = 512 and 256 at M = 64)
  static constexpr int NS = M == 128 ? 6 : (C == 512) ? 3 : (C == 256 ? 6 : 8);
  static constexpr uint32_t kPBytes = M * 128;   // P tile: M rows x 64 keys (bf16)
  static constexpr int SP = M == 128 ? 3 : kSP;    // S / P buffers
  static constexpr uint32_t kv_off = 0;
  static constexpr uint32_t p_off = kv_off + NS * NKB * kTileBytes;
  // M = 128: a ring of two unit slots filled by the loaders -- the unit's Q
  // rows [128][C] bf16 (chunks swizzled by row) and its RoPE table [8
  // queries][cos 32 | sin 32] fp32
  static constexpr uint32_t kQStage = 128u * C * 2, kRope = 8u * 64 * 4;
  static constexpr uint32_t q_off = p_off + SP * kPBytes;
  static constexpr uint32_t r_off = q_off + (M == 128 ? 2 * kQStage : 0u);
  static constexpr uint32_t bar_off = r_off + (M == 128 ? 2 * kRope : 0u);
  static constexpr uint32_t misc_off = bar_off + 512;
  static constexpr uint32_t bytes = misc_off + 8192 + 1024;  // + alignment slack
  // tensor memory.  M = 64: O in lane-half 0, columns [0, C); in lane-half 1
  // S buffers 0 and 1 at columns [0, 128), Q (bf16, two per column) at
  // [q_col, q_col + C/2), the lanes of S as the A operand of S = Q K^T needs,
  // and S buffer 2 after Q.  M = 128: O accumulators at [0, C) and [C, 2C),
  // three S buffers from column 2C, Q at [2C + 192, 2C + 192 + C/2).
  static constexpr uint32_t tmem_cols = 512;
  static constexpr uint32_t o_cols = M == 128 ? 2 * C : C;
  static constexpr uint32_t q_col = M == 64 ? 2 * KT : o_cols + SP * KT;
  static constexpr uint32_t s_lane = M == 64 ? 16 : 0;   // lane offset of S and Q in each quarter
  static_assert(q_col + C / 2 + (M == 64 ? KT : 0) <= tmem_cols, "S buffers and Q exceed tensor memory");
  static_assert(bytes <= 227 * 1024, "shared memory");
  static constexpr __host__ __device__ uint32_t s_col(int b) {
    return M == 128 ? o_cols + b * KT : (b < 2 ? b * KT : q_col + C / 2);
  }
};

// Trace counters (cycles, summed over CTAs) of the tensor-core kernel's waits.
enum TraceSlot {
  TR_P_QEMPTY, TR_P_KVEMPTY, TR_M_QFULL, TR_M_KVFULL, TR_M_SEMPTY, TR_M_PFULL, TR_M_OEMPTY,
  TR_S_SFULL, TR_S_PBUF, TR_S_RESCALE, TR_S_EPI_WAIT, TR_S_TILE, TR_S_EPI, TR_TOTAL, TR_RESCALES, TR_UNITS,
  TR_TILES, TR_P_ISSUE, TR_S_MERGE_READY, TR_S_MERGE_FULL, TR_S_PUSH, TR_S_WEIGHTS, TR_S_MERGE_LOOP,
  // timeline of each CTA's first unit (ns, summed over CTAs): setup, until the
  // first S, the tiles, the epilogue/merge, until exit; then the earliest
  // entry (stored inverted) and the latest exit over all CTAs, and the CTA count
  TR_T_SETUP, TR_T_FIRST_S, TR_T_TILES, TR_T_EPI, TR_T_EXIT, TR_T_ENTRY_INV, TR_T_EXIT_MAX, TR_T_CTAS, TR_COUNT
};
__device__ unsigned long long g_attn_trace[32];

// Named barrier over the 4 softmax warps (warps 0-3).
__device__ __forceinline__ void softmax_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxWarps * 32) : "memory");
}

// ---------------------------------------------------------------- cluster merge
// With nsplit <= 8 the splits of one query form a thread-block cluster (one
// unit per CTA).  CTA `sp` owns output columns [sp*per, (sp+1)*per).  After
// its last P.V, each CTA stages its unnormalised O rows (bf16) and per-row
// (max, sum) as one block per owner, then one thread sends every other
// owner its block with a bulk shared-to-distributed-shared copy that
// completes on the owner's mg_full barrier.  Copies into a peer start only
// once every CTA of the cluster has reported (mg_ready) that its tiles are
// done, since the blocks overlay the Q and key-tile buffers.  The owner
// forms  o = sum_i 2^{m_i-M} O_i / (sum_i 2^{m_i-M} l_i + 2^{sink-M})  for its
// columns, applies the inverse RoPE and stores bf16.  The 4 softmax warps and
// the 8 load warps (idle by then) share the work: 3 warps per TMEM lane
// quarter read O, 384 threads merge.  All waits are bounded.
__host__ __device__ constexpr int merge_cols(int C, int ns) { return ((C / ns + 15) / 16) * 16; }
__host__ __device__ constexpr int merge_pitch(int C, int ns) { return merge_cols(C, ns) + 8; }   // bf16 elements
// one owner's block: O [64][pitch] bf16, then (max, sum) [64] float2
__host__ __device__ constexpr uint32_t merge_blk(int C, int ns) { return 64u * merge_pitch(C, ns) * 2 + 64 * 8; }
// staged blocks [ns], received blocks [ns] (own slot unused)
__host__ __device__ constexpr uint32_t merge_bytes(int C, int ns) { return 2u * ns * merge_blk(C, ns); }
template <int C>
__host__ __device__ constexpr bool merge_fits() {
  for (int ns = 2; ns <= kMaxClusterSplits; ++ns)
    if (merge_bytes(C, ns) > Layout<C>::p_off) return false;
  return true;
}
constexpr int kMergeThreads = (kSoftmaxWarps + kProdWarps) * 32;

// Bounded rendezvous of the 12 merge warps (softmax warps 0-3, load warps
// 5-12) on a one-shot mbarrier that counts one arrival per warp.
__device__ __forceinline__ bool merge_sync(uint64_t *b, int *status) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(b));
  return mbar_wait(smem_u32(b), 0, status);
}
__device__ __forceinline__ void bulk_s2c(uint32_t dst_cluster, uint32_t src, uint32_t bytes, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(src), "r"(bytes), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Called by the 12 merge warps once the softmax warps have written every
// staged block's (max, sum) and all have waited for the unit's last P.V.
template <int C>
__device__ __forceinline__ bool cluster_merge(const AttendParams &p, uint8_t *smem, Bars *bars, uint32_t tmem,
                                              int nt, int sp, int b, int qi, const float *rope_cs,
                                              unsigned long long *trace) {
  static_assert(merge_fits<C>(), "merge buffers overlap the P buffers");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (warp < kSoftmaxWarps ? warp : warp - 1) * 32 + lane;   // 0..383
  const int quarter = warp & 3, third = warp < kSoftmaxWarps ? 0 : 1 + (warp - kProdWarp0) / 4;
  const int hl = lane & 15, half = lane >> 4;
  const int r = quarter * 16 + hl;
  const int ns = p.nsplit;
  const int per = merge_cols(C, ns), pitch = merge_pitch(C, ns);
  const uint32_t blk = merge_blk(C, ns);
  uint8_t *stage = smem;                      // [ns] blocks
  uint8_t *recv = smem + ns * blk;            // [ns] blocks
  long long tw = trace ? clock64() : 0;
  // ---- stage O (bf16), 16 columns per TMEM load
  if (nt > 0) {
    tc_fence_after();
    const uint32_t tq = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int k = third; k < C / 32; k += 3) {
      uint32_t ov[16];
      tmem_ld_16x32bx2_x16<C / 2>(tq + 16 * k, ov);
      tmem_ld_wait();
      const int col0 = half * (C / 2) + 16 * k;
      const int owner = col0 / per;
      __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(stage + owner * blk) + r * pitch + (col0 - owner * per);
      uint4 w0, w1;
      w0.x = pack_bf16x2(__uint_as_float(ov[0]), __uint_as_float(ov[1]));
      w0.y = pack_bf16x2(__uint_as_float(ov[2]), __uint_as_float(ov[3]));
      w0.z = pack_bf16x2(__uint_as_float(ov[4]), __uint_as_float(ov[5]));
      w0.w = pack_bf16x2(__uint_as_float(ov[6]), __uint_as_float(ov[7]));
      w1.x = pack_bf16x2(__uint_as_float(ov[8]), __uint_as_float(ov[9]));
      w1.y = pack_bf16x2(__uint_as_float(ov[10]), __uint_as_float(ov[11]));
      w1.z = pack_bf16x2(__uint_as_float(ov[12]), __uint_as_float(ov[13]));
      w1.w = pack_bf16x2(__uint_as_float(ov[14]), __uint_as_float(ov[15]));
      reinterpret_cast<uint4 *>(dst)[0] = w0;
      reinterpret_cast<uint4 *>(dst)[1] = w1;
    }
    tc_fence_before();
  }
  fence_proxy_async();   // staged blocks are read by the bulk-copy engine
  if (!merge_sync(&bars->mg_stage, p.status)) return false;
  if (trace) { const long long t = clock64(); trace[2] += t - tw; tw = t; }
  // ---- every CTA's tiles are done -> send each owner its block
  bool sent = false;
  if (mt == 0) {
    for (int j = 0; j < ns; ++j) mbar_arrive_cluster(cluster_map(smem_u32(&bars->mg_ready), j));
    if (mbar_wait_cluster(smem_u32(&bars->mg_ready), 0, p.status)) {
      for (int j = 0; j < ns; ++j)
        if (j != sp)
          bulk_s2c(cluster_map(smem_u32(recv + sp * blk), j), smem_u32(stage + j * blk), blk,
                   cluster_map(smem_u32(&bars->mg_full), j));
      bulk_commit();
      sent = true;
    }
  }
  if (trace) { const long long t = clock64(); trace[0] += t - tw; tw = t; }
  bool ok = mbar_wait_cluster(smem_u32(&bars->mg_full), 0, p.status);
  if (trace) { const long long t = clock64(); trace[1] += t - tw; tw = t; }
  if (ok) {
    auto ml_of = [&](int i, int row) -> float2 {
      const uint8_t *base = (i == sp ? stage + i * blk : recv + i * blk);
      return reinterpret_cast<const float2 *>(base + 64u * pitch * 2)[row];
    };
    // ---- this CTA's columns of every head row, 8 columns per item; each item
    // derives its row's merge weights from the (max, sum) pairs itself
    const int c_lo = min(C, sp * per), c_hi = min(C, c_lo + per);
    const int ngr = (c_hi - c_lo) / 8;
    for (int it = mt; it < 64 * ngr; it += kMergeThreads) {
      const int row = it / ngr, cg = c_lo + 8 * (it % ngr);
      if (row >= p.n_h) continue;
      const float sink2 = p.sink[row] * kLog2e;
      float mi[kMaxClusterSplits], li[kMaxClusterSplits];
      float M = sink2;
#pragma unroll
      for (int i = 0; i < kMaxClusterSplits; ++i) {
        const float2 v = i < ns ? ml_of(i, row) : make_float2(-INFINITY, 0.f);
        mi[i] = v.x;
        li[i] = v.y;
        if (v.y > 0.f) M = fmaxf(M, v.x);
      }
      float den = exp2f(sink2 - M);
#pragma unroll
      for (int i = 0; i < kMaxClusterSplits; ++i) {
        mi[i] = li[i] > 0.f ? exp2f(mi[i] - M) : 0.f;   // now the unnormalised weight
        den += mi[i] * li[i];
      }
      const float inv = 1.f / den;
      float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < ns; ++i) {
        const float w = mi[i] * inv;
        if (w == 0.f) continue;
        const uint8_t *base = (i == sp ? stage + i * blk : recv + i * blk);
        const uint4 v = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(base) +
                                                         row * pitch + (cg - c_lo));
        o[0] += w * bf16_lo(v.x); o[1] += w * bf16_hi(v.x);
        o[2] += w * bf16_lo(v.y); o[3] += w * bf16_hi(v.y);
        o[4] += w * bf16_lo(v.z); o[5] += w * bf16_hi(v.z);
        o[6] += w * bf16_lo(v.w); o[7] += w * bf16_hi(v.w);
      }
      if (cg + 8 > C - p.rd) {
#pragma unroll
        for (int x = 0; x < 8; x += 2) {
          const int col = cg + x;
          if (col >= C - p.rd) {
            const int pi = (col - (C - p.rd)) / 2;
            const float cs = rope_cs[pi], sn = rope_cs[32 + pi];
            const float aa = o[x], bb = o[x + 1];
            o[x] = aa * cs + bb * sn;
            o[x + 1] = -aa * sn + bb * cs;
          }
        }
      }
      uint4 w4;
      w4.x = pack_bf16x2(o[0], o[1]); w4.y = pack_bf16x2(o[2], o[3]);
      w4.z = pack_bf16x2(o[4], o[5]); w4.w = pack_bf16x2(o[6], o[7]);
      *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.o) +
                                 (((long long)b * p.n_q + qi) * p.n_h + row) * C + cg) = w4;
    }
    if (trace) trace[4] += clock64() - tw;
  }
  // the staged blocks must have been read before this CTA leaves
  if (sent) bulk_wait_read_all();
  return ok;
}

template <int C, int M, bool TRACE, bool MIX>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc(AttendParams p, int n_units) {
  using L = Layout<C, M>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  Bars *bars = reinterpret_cast<Bars *>(smem + L::bar_off);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::misc_off);
  double *freq = reinterpret_cast<double *>(smem + L::misc_off + 8);      // [32]
  float *rope_all = reinterpret_cast<float *>(smem + L::misc_off + 512);   // M = 64: [4 warps][64]: cos, sin
  float *xch = reinterpret_cast<float *>(smem + L::misc_off + 4608);       // M = 128: (max, sum) [8 warps][32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // warp roles: softmax warps first, then the MMA warp, then the loaders.
  // M = 128: two softmax warps per TMEM lane quarter (each takes 32 of a
  // tile's 64 keys and half of the O columns) and 4 loaders (c <= 256)
  constexpr int SMW = M == 128 ? 8 : kSoftmaxWarps;
  constexpr int MMAW = SMW;
  constexpr int PW0 = SMW + 1;
  constexpr int PT = (M == 128 ? 4 : kProdWarps) * 32;
  static_assert((SMW + 1) * 32 + PT == kThreads, "warp roles");
  // S / P buffers and how many S tiles the MMA issue runs ahead of P.V
  constexpr int SP = L::SP;
  constexpr int LA = M == 128 ? 2 : kLookahead;
  const unsigned long long st_entry = global_ns();
  auto bar = [&](uint64_t &b) { return smem_u32(&b); };
  unsigned long long tr[TR_COUNT];
  if (TRACE) for (int i = 0; i < TR_COUNT; ++i) tr[i] = 0;
  const long long t_start = TRACE ? clock64() : 0;
  unsigned long long ts[6] = {0, 0, 0, 0, 0, 0};   // timeline stamps (thread 0, first unit)
  if (TRACE && threadIdx.x == 0) ts[0] = global_ns();
  // wait on an mbarrier, adding the cycles spent to trace slot `slot`
  auto twait = [&](uint32_t b, uint32_t par, int slot) -> bool {
    if (!TRACE) return mbar_wait(b, par, p.status);
    const long long t0 = clock64();
    const bool ok = mbar_wait(b, par, p.status);
    tr[slot] += clock64() - t0;
    return ok;
  };
  // loaders wait for free stages sleeping between polls
  auto twait_sleep = [&](uint32_t b, uint32_t par, int slot) -> bool {
    if (!TRACE) return mbar_wait_sleep(b, par, p.status);
    const long long t0 = clock64();
    const bool ok = mbar_wait_sleep(b, par, p.status);
    tr[slot] += clock64() - t0;
    return ok;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(bars->q_full), SMW);
    mbar_init(bar(bars->q_empty), 1);
    mbar_init(bar(bars->o_empty), SMW);
    mbar_init(bar(bars->mma_done), 1);
    for (int i = 0; i < L::NS; ++i) {
      mbar_init(bar(bars->kv_full[i]), PT);
      mbar_init(bar(bars->kv_empty[i]), 1);
    }
    for (int i = 0; i < SP; ++i) {
      mbar_init(bar(bars->s_full[i]), 1);
      mbar_init(bar(bars->s_empty[i]), M == 128 ? 1 : SMW);   // M = 128: released by the MMA after P.V
      mbar_init(bar(bars->p_full[i]), SMW);
      mbar_init(bar(bars->pv_done[i]), 1);
    }
    if (M == 128) {
      for (int i = 0; i < 4; ++i) mbar_init(bar(bars->pair[i]), 2);
      // per loader thread: its Q copies landed (cp.async arrive) and its RoPE stores
      for (int i = 0; i < 2; ++i) mbar_init(bar(bars->us_full[i]), 2 * PT);
      for (int i = 0; i < 2; ++i) mbar_init(bar(bars->us_empty[i]), SMW);
    }
    if (p.cluster) {
      mbar_init(bar(bars->mg_ready), p.nsplit);
      mbar_init(bar(bars->mg_full), 1);
      mbar_init(bar(bars->mg_stage), kMergeThreads / 32);
    }
    mbar_fence_init();
  }
  if (warp == MMAW) {
    tmem_alloc(smem_u32(tmem_slot), L::tmem_cols);
    tmem_relinquish();
  }
  if (threadIdx.x < p.rd / 2) freq[threadIdx.x] = p.rope_freq[threadIdx.x];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // peers arrive on this CTA's merge barriers only after every CTA initialised its own
  if (p.cluster) {
    if (threadIdx.x == 0) mbar_arrive_expect_tx(bar(bars->mg_full), (p.nsplit - 1) * merge_blk(C, p.nsplit));
    cluster_sync();
  }
  pdl_wait();   // indices, caches and queries of the previous launch are complete
  const unsigned long long st_ready = global_ns();
  if (TRACE && threadIdx.x == 0) ts[1] = global_ns();

  if (warp >= PW0) {
    // ------------------------------------------------------------ loads
    // Q: 2-D tiled TMA (thread 0).  Key rows: cp.async by 8 warps, 16-byte
    // chunks placed at their 128B-swizzled positions; every thread resolves
    // all of its row addresses for the tile first (independent index loads),
    // then issues its copies and arms the stage barrier to complete when they
    // land.
    [&]() {
    constexpr int NKB = C / 64;
    constexpr int CPR = C / 8;                  // 16-byte chunks per row
    constexpr int RPP = PT / CPR;               // rows per pass
    constexpr int NR = KT / RPP;                // rows per thread per tile
    const int pt = threadIdx.x - PW0 * 32;
    const int chunk = pt % CPR, prow = pt / CPR;
    const uint32_t kb_off = (chunk / 8) * kTileBytes;
    const int cc = chunk % 8;
    uint32_t g = 0, lv = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const Unit x = unit_of(p, u);
      const int b = x.b, qi = x.qi0;
      const KeySet ks = group_key_set(p, x.qg);
      int j0, nt;
      split_range(ks, p.nsplit, x.sp, j0, nt);
      if (nt == 0) continue;
      if constexpr (M == 128) {
        // the unit's slot: thread pt copies Q row pt (head pt % n_h of query
        // pt / n_h), 16-byte chunk i to position i ^ (pt & 7), and computes
        // RoPE entries pt and pt + 128 of the unit's [G][rd/2] table
        const int slot = lv & 1;
        if (!twait_sleep(bar(bars->us_empty[slot]), ((lv >> 1) & 1) ^ 1, TR_P_QEMPTY)) return;
        const int qg = pt / p.n_h, hq = pt - qg * p.n_h;
        const bool live = qi + qg < p.n_q;
        const char *src = reinterpret_cast<const char *>(
            reinterpret_cast<const __nv_bfloat16 *>(p.q) +
            (live ? (((long long)b * p.n_q + qi + qg) * p.n_h + hq) * C : 0));
        const uint32_t qrow = sbase + L::q_off + slot * L::kQStage + pt * (C * 2);
#pragma unroll
        for (int i = 0; i < C / 8; ++i) cp_async16(qrow + ((i ^ (pt & 7)) << 4), src + 16 * i, live ? 16 : 0);
        cp_async_arrive_noinc(bar(bars->us_full[slot]));
        float *rope = reinterpret_cast<float *>(smem + L::r_off + slot * L::kRope);
        for (int e = pt; e < p.G * 32; e += PT) {
          const int gq = e >> 5, i = e & 31;
          if (i < p.rd / 2) {
            double ang = (double)(p.start_pos + qi + gq) * freq[i];
            ang -= 6.283185307179586476925286766559 * rint(ang * 0.15915494309189533576888376337251);
            float sn, cs;
            __sincosf((float)ang, &sn, &cs);   // |ang| <= pi: error below 1e-6
            rope[gq * 64 + i] = cs;
            rope[gq * 64 + 32 + i] = sn;
          }
        }
        mbar_arrive(bar(bars->us_full[slot]));
        ++lv;
      }
      if (p.csa && pt < 32) {
        // index lists: this unit's into L1 (read tile by tile below), the next
        // unit's of this CTA into L2
        const int32_t *il = p.idx + ((long long)b * p.n_q + qi) * p.k;
        const int lines = (p.k * 4 + 127) / 128;
        for (int x = pt; x < lines; x += 32) asm volatile("prefetch.global.L1 [%0];" ::"l"(il + 32 * x));
        const int un = u + gridDim.x;
        if (un < n_units) {
          const int32_t *nl = p.idx + (long long)fdiv(un, p.fd_nsplit) * p.k;
          for (int x = pt; x < lines; x += 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(nl + 32 * x));
        }
      }
      // masked slots read a real row of a real tensor (cap is 0 when kv_comp is absent)
      const __nv_bfloat16 *cbase = reinterpret_cast<const __nv_bfloat16 *>(
          p.kv_comp ? p.kv_comp : (p.kv_win ? p.kv_win : p.q));
      const __nv_bfloat16 *wbase = p.kv_win ? reinterpret_cast<const __nv_bfloat16 *>(p.kv_win) : cbase;
      if (MIX) {
        // mixed-precision records: a thread whose chunk holds FP8 codes loads
        // its 8 codes and their block scale for all of its rows (independent
        // loads, all in flight), waits for the stage, and writes the bf16
        // values code x scale; a thread of the bf16 RoPE channels copies them
        const uint8_t *crec = reinterpret_cast<const uint8_t *>(p.kv_comp ? p.kv_comp : (p.kv_win ? p.kv_win : p.q));
        const uint8_t *wrec = p.kv_win ? reinterpret_cast<const uint8_t *>(p.kv_win) : crec;
        const int ch0 = chunk * 8, nq = C - p.rd;
        const bool code = ch0 < nq;
        const int col_off = code ? ch0 : nq + 2 * (ch0 - nq);
        const int sc_off = C + p.rd + 4 * (ch0 / 64);
        for (int j = 0; j < nt; ++j, ++g) {
          const int st = g % L::NS;
          const uint32_t tile = sbase + L::kv_off + st * NKB * kTileBytes + kb_off;
          if (code) {
            uint2 cw[NR];
            float sc[NR];
#pragma unroll
            for (int i = 0; i < NR; ++i) {
              const int kk = (j0 + j) * KT + prow + i * RPP;
              bool v;
              const int row = slot_row(p, ks, b, qi, kk, v);
              const uint8_t *rp = (kk < ks.nw4 ? wrec : crec) + (long long)row * p.rec;
              cw[i] = __ldg(reinterpret_cast<const uint2 *>(rp + col_off));
              sc[i] = __ldg(reinterpret_cast<const float *>(rp + sc_off));
            }
            if (!twait_sleep(bar(bars->kv_empty[st]), ((g / L::NS) & 1) ^ 1, TR_P_KVEMPTY)) return;
#pragma unroll
            for (int i = 0; i < NR; ++i) {
              const uint32_t w2[2] = {cw[i].x, cw[i].y};
              uint32_t o[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const uint32_t pair = (w2[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
                const float2 f = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)pair, __NV_E4M3)));
                o[h] = pack_bf16x2(f.x * sc[i], f.y * sc[i]);
              }
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(tile + sw128_off(prow + i * RPP, cc)),
                           "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                           : "memory");
            }
            fence_proxy_async();   // the tensor cores read the tile through the async proxy
            mbar_arrive(bar(bars->kv_full[st]));
          } else {
            const uint8_t *src8[NR];
#pragma unroll
            for (int i = 0; i < NR; ++i) {
              const int kk = (j0 + j) * KT + prow + i * RPP;
              bool v;
              const int row = slot_row(p, ks, b, qi, kk, v);
              src8[i] = (kk < ks.nw4 ? wrec : crec) + (long long)row * p.rec + col_off;
            }
            if (!twait_sleep(bar(bars->kv_empty[st]), ((g / L::NS) & 1) ^ 1, TR_P_KVEMPTY)) return;
#pragma unroll
            for (int i = 0; i < NR; ++i) cp_async16(tile + sw128_off(prow + i * RPP, cc), src8[i], 16);
            cp_async_arrive_noinc(bar(bars->kv_full[st]));
          }
        }
        continue;
      }
      for (int j = 0; j < nt; ++j, ++g) {
        const int st = g % L::NS;
        const __nv_bfloat16 *src[NR];
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const int kk = (j0 + j) * KT + prow + i * RPP;
          bool v;
          const int row = slot_row(p, ks, b, qi, kk, v);
          src[i] = (kk < ks.nw4 ? wbase : cbase) + (long long)row * C + chunk * 8;
        }
        if (!twait_sleep(bar(bars->kv_empty[st]), ((g / L::NS) & 1) ^ 1, TR_P_KVEMPTY)) return;
        const uint32_t tile = sbase + L::kv_off + st * NKB * kTileBytes + kb_off;
#pragma unroll
        for (int i = 0; i < NR; ++i) cp_async16(tile + sw128_off(prow + i * RPP, cc), src[i], 16);
        cp_async_arrive_noinc(bar(bars->kv_full[st]));
      }
    }
    }();
    cp_async_wait_all();
    if (M == 64 && p.cluster) {
      // one unit per CTA: join the merge once its last P.V has landed
      const Unit x = unit_of(p, blockIdx.x);
      const int b = x.b, qi = x.qi0, sp = x.sp;
      const KeySet ks = group_key_set(p, x.qg);
      int j0, nt;
      split_range(ks, p.nsplit, sp, j0, nt);
      // the unit's last P.V has landed once the MMA warp's final commit has
      // (a parity wait on pv_done is only meaningful one phase ahead of the
      // last phase this thread has seen, and this thread has seen none)
      bool ok = true;
      if (nt > 0) ok = mbar_wait(bar(bars->mma_done), 0, p.status);
      if (ok) {
        // the softmax warps' (max, sum) writes and RoPE table are ordered by the merge barrier
        cluster_merge<C>(p, smem, bars, tmem, nt, sp, b, qi, rope_all, nullptr);
      }
    }
  } else if (warp == MMAW) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(M, KT, 0, 0);
      constexpr int NPV = C < 256 ? C : 256;
      constexpr uint32_t IDESC_PV = idesc_bf16(M, NPV, 0, 1);
      const uint32_t tS = tmem + (L::s_lane << 16);
      uint32_t g = 0, iq = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t gg, bool first) -> bool {
        const int st = gg % SP;               // S / P buffer
        const int kst = gg % L::NS;            // key-tile stage
        if (!twait(bar(bars->p_full[st]), (gg / SP) & 1, TR_M_PFULL)) return false;
        if (first && !twait(bar(bars->o_empty), (iq & 1) ^ 1, TR_M_OEMPTY)) return false;
        tc_fence_after();
        const uint32_t pa = sbase + L::p_off + st * L::kPBytes;
        const uint32_t va = sbase + L::kv_off + kst * L::NKB * kTileBytes;
        const uint64_t pd = sdesc_sw128(pa, 16, 1024);
        const uint64_t vd = sdesc_sw128(va, kTileBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          // M = 128: keys [0, 32) of the tile into O accumulator 0, [32, 64) into 1
          const uint32_t o_acc = M == 128 ? (kk >> 1) * C : 0;
          const bool reset = first && (M == 128 ? (kk & 1) == 0 : kk == 0);
#pragma unroll
          for (int nh = 0; nh < C / NPV; ++nh) {
            const uint64_t voff = (nh * (NPV / 64) * kTileBytes + kk * 16 * 128) >> 4;
            if constexpr (M == 128) {
              // P (bf16) in the tile's S columns: keys [32h, 32h + 32) of
              // every row at columns s_col + 32h .. + 16, the A operand
              const uint32_t pa_t = tS + L::s_col(st) + 32 * (kk >> 1) + 8 * (kk & 1);
              umma_bf16_ts(tmem + o_acc + nh * NPV, pa_t, vd + voff, IDESC_PV, reset ? 0u : 1u);
            } else {
              umma_bf16(tmem + o_acc + nh * NPV, pd + ((kk * 32) >> 4), vd + voff, IDESC_PV, reset ? 0u : 1u);
            }
          }
        }
        umma_commit(bar(bars->kv_empty[kst]));
        umma_commit(bar(bars->pv_done[st]));
        if (M == 128) umma_commit(bar(bars->s_empty[st]));   // the S / P columns are free
        return true;
      };
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit x = unit_of(p, u);
        const KeySet ks = group_key_set(p, x.qg);
        int j0, nt;
        split_range(ks, p.nsplit, x.sp, j0, nt);
        if (nt == 0) continue;
        if (!twait(bar(bars->q_full), iq & 1, TR_M_QFULL)) { ok = false; break; }
        fence_proxy_async();
        tc_fence_after();
        // S of tile j, then P.V of tile j - LA; the unit's last P.Vs
        // are issued before the next unit's Q is awaited (its epilogue waits
        // for them)
        int npv = 0;                           // P.Vs of this unit issued
        for (int j = 0; j < nt && ok; ++j) {
          const uint32_t gj = g + j;
          const int st = gj % SP;
          const uint32_t ph = (gj / SP) & 1;
          const int kst = gj % L::NS;
          if (!twait(bar(bars->kv_full[kst]), (gj / L::NS) & 1, TR_M_KVFULL) ||
              !twait(bar(bars->s_empty[st]), ph ^ 1, TR_M_SEMPTY)) {
            ok = false;
            break;
          }
          fence_proxy_async();
          tc_fence_after();
          // K descriptor advances by constant offsets (16-byte units in the low
          // field); Q (A operand, tensor memory) by 8 columns = 16 bf16 per step
          const uint64_t kd = sdesc_sw128(sbase + L::kv_off + kst * L::NKB * kTileBytes, 16, 1024);
          const uint32_t sd = tS + L::s_col(st);
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk) {
            const uint64_t off = ((kk / 4) * kTileBytes + (kk % 4) * 32) >> 4;
            umma_bf16_ts(sd, tS + L::q_col + 8 * kk, kd + off, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(bars->s_full[st]));
          if (j == nt - 1) umma_commit(bar(bars->q_empty));
          if (j >= LA) {
            if (!issue_pv(g + npv, npv == 0)) ok = false;
            ++npv;
          }
        }
        for (; ok && npv < nt; ++npv)
          if (!issue_pv(g + npv, npv == 0)) ok = false;
        g += nt;
        ++iq;
      }
      umma_commit(bar(bars->mma_done));
      mbar_wait(bar(bars->mma_done), 0, p.status);
    }
    __syncwarp();
  } else if constexpr (M == 128) {
    // ------------------------------------------------------------ softmax + epilogue, 128 rows
    // Query groups on 128 rows (c = 128).  Warps w and w + 4 share TMEM lane
    // quarter w % 4: thread (warp, lane) owns row r = (w % 4) * 32 + lane --
    // head rh of query rg of the group -- for the keys [32 hf, 32 hf + 32) of
    // every tile, hf = w / 4, with its own running max and sum and its own O
    // accumulator (P.V of those keys).  At the end of a unit the two warps
    // exchange (max, sum) and each combines both accumulators for the O
    // columns [hf C/2, (hf + 1) C/2).  A warp's rows belong to one query
    // (n_h >= 32) or two (n_h = 16).
    [&]() {
    const int q4 = warp & 3, hf = warp >> 2;
    const int r = q4 * 32 + lane;
    const int rg = r / p.n_h, rh = r - rg * p.n_h;
    const float zs = p.scale * kLog2e;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tmem + lane_base + hf * C;   // this warp's O accumulator
    constexpr int CH = C / 2;             // O columns (and Q dims) of this warp
    constexpr int NQC = CH / 8;           // 16-byte chunks of a half row
    const int col_lo = hf * CH;
    // bounded rendezvous of the two warps of this lane quarter: their shared
    // memory writes before it are visible to both after it
    uint32_t npair = 0;
    auto pair_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bars->pair[q4]));
      return mbar_wait(bar(bars->pair[q4]), (npair++) & 1, p.status);
    };
    // Q of unit slot lvq (staged by the loaders: row r's 16-byte chunk i at
    // position i ^ (r & 7)) into tensor memory, row r, columns q_col + col_lo/2 ..,
    // once the current unit's last S has been read
    uint32_t nq = 0;                      // Q writes so far (q_empty parity)
    auto write_q = [&](uint32_t lvq) -> bool {
      const int slot = lvq & 1;
      if (!twait(bar(bars->us_full[slot]), (lvq >> 1) & 1, TR_P_QEMPTY)) return false;
      if (nq > 0 && !twait(bar(bars->q_empty), (nq - 1) & 1, TR_P_QEMPTY)) return false;
      tc_fence_after();
      const uint32_t qrow = sbase + L::q_off + slot * L::kQStage + r * (C * 2);
      uint32_t v[NQC * 4];
#pragma unroll
      for (int i = 0; i < NQC; ++i)
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v[4 * i]), "=r"(v[4 * i + 1]), "=r"(v[4 * i + 2]), "=r"(v[4 * i + 3])
                     : "r"(qrow + (((hf * NQC + i) ^ (r & 7)) << 4))
                     : "memory");
      const uint32_t tq = tmem + lane_base + L::q_col + col_lo / 2;
#pragma unroll
      for (int y = 0; y < NQC / 4; ++y) tmem_st_32x32b_x16(tq + 16 * y, *reinterpret_cast<const uint32_t(*)[16]>(&v[16 * y]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bars->q_full));
      ++nq;
      return true;
    };
    auto next_unit = [&](int u0) -> int {
      for (int uu = u0 + gridDim.x; uu < n_units; uu += gridDim.x) {
        int a0, an;
        const Unit xu = unit_of(p, uu);
        split_range(group_key_set(p, xu.qg), p.nsplit, xu.sp, a0, an);
        if (an > 0) return uu;
      }
      return -1;
    };
    int q_ready_u = -1;
    uint32_t g = 0, lv = 0;               // tiles and units (with tiles) so far
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const long long tu0 = TRACE ? clock64() : 0;
      const Unit ux = unit_of(p, u);
      const int b = ux.b, qi = ux.qi0;
      const bool live = qi + rg < p.n_q;
      const KeySet ks = group_key_set(p, ux.qg);
      int j0, nt;
      split_range(ks, p.nsplit, ux.sp, j0, nt);
      // this row's keys among the group's slots: window slots [w_lo, w_hi)
      // (tokens tq - w + 1 .. tq) and entry slots [nw4, c_hi)
      const int tq = p.start_pos + qi + rg;
      const int w_lo = max(0, tq - p.w + 1 - ks.t0), w_hi = p.w > 0 ? min(tq - ks.t0 + 1, ks.nw) : 0;
      const int c_hi = ks.nw4 + fdiv(tq + 1, p.fd_m);
      if (nt > 0 && q_ready_u != u) {
        if (!write_q(lv)) return;
        q_ready_u = u;
      }
      const int un = nt > 0 ? next_unit(u) : -1;
      __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) +
                            (live ? (((long long)b * p.n_q + qi + rg) * p.n_h + rh) * C : 0);
      if (nt == 0) {
        if (live)
          for (int col = col_lo; col < col_lo + CH; col += 8)
            *reinterpret_cast<uint4 *>(orow + col) = make_uint4(0, 0, 0, 0);
        continue;
      }
      // this row's query's RoPE table in the unit's slot (inverse rotation in the epilogue)
      const float *rope_cs = reinterpret_cast<const float *>(smem + L::r_off + (lv & 1) * L::kRope) + rg * 64;
      // running max (log2 units; -inf until a valid key is seen) and sum
      float m_used = -INFINITY, l = 0.f;
      if (TRACE) tr[TR_S_TILE] += clock64() - tu0;   // the unit's setup
      if (TRACE) { tr[TR_UNITS] += 1; tr[TR_TILES] += nt; }
      for (int j = 0; j < nt; ++j) {
        const uint32_t gj = g + j;
        const int st = gj % SP;
        const uint32_t ph = (gj / SP) & 1;
        if (!twait(bar(bars->s_full[st]), ph, TR_S_SFULL)) return;
        if (TRACE && threadIdx.x == 0 && j == 0 && ts[2] == 0) ts[2] = global_ns();
        // sub-phase cycles of the tile (the merge slots are unused at M = 128)
        long long tp = TRACE ? clock64() : 0;
        auto phase = [&](int slot) {
          if (TRACE) {
            const long long t1 = clock64();
            tr[slot] += t1 - tp;
            tp = t1;
          }
        };
        tc_fence_after();
        uint32_t sv[32];
        tmem_ld_32x32b_x16(tmem + lane_base + L::s_col(st) + 32 * hf, *reinterpret_cast<uint32_t(*)[16]>(&sv[0]));
        tmem_ld_32x32b_x16(tmem + lane_base + L::s_col(st) + 32 * hf + 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[16]));
        tmem_ld_wait();
        phase(TR_S_MERGE_READY);
        // this row's valid keys among the warp's 32
        const int kb = (j0 + j) * KT + 32 * hf;
        const uint32_t vm = range_bits(kb, w_lo, w_hi) | range_bits(kb, ks.nw4, c_hi);
        float z[32];
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          z[x] = ((vm >> x) & 1u) ? __uint_as_float(sv[x]) * zs : -INFINITY;
          mx[x & 3] = fmaxf(mx[x & 3], z[x]);
        }
        const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        phase(TR_S_MERGE_FULL);
        // lazy rescaling: the max moves only when it grows by more than 8
        bool need = false;
        float alpha = 1.f;
        if (tmax != -INFINITY && (m_used == -INFINITY || tmax > m_used + 8.f)) {
          if (m_used != -INFINITY) {   // before the first valid key O and l are 0
            need = true;
            alpha = ex2_approx(m_used - tmax);
            l *= alpha;
          }
          m_used = tmax;
        }
        if (__any_sync(0xffffffffu, need)) {
          // rescale this warp's O accumulator after the P.V of the previous tile lands
          const uint32_t gp = gj - 1;
          if (TRACE) tr[TR_RESCALES] += 1;
          if (!twait(bar(bars->pv_done[gp % SP]), (gp / SP) & 1, TR_S_RESCALE)) return;
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < C; c0 += 16) {
            uint32_t ov[16];
            tmem_ld_32x32b_x16(tO + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 16; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
            tmem_st_32x32b_x16(tO + c0, ov);
          }
          tmem_st_wait();
        }
        const float m_eff = m_used == -INFINITY ? 0.f : m_used;
        float ps[2] = {0.f, 0.f};
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float p0 = ex2_approx(z[x] - m_eff), p1 = ex2_approx(z[x + 1] - m_eff);
          ps[(x >> 1) & 1] += p0 + p1;
          pk[x / 2] = pack_bf16x2(p0, p1);
        }
        l += ps[0] + ps[1];
        phase(TR_S_PUSH);
        // P (bf16) over the first 16 of this warp's 32 S columns of the tile
        // (already read); the P.V reads it from tensor memory
        tmem_st_32x32b_x16(tmem + lane_base + L::s_col(st) + 32 * hf, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bars->p_full[st]));
        phase(TR_S_WEIGHTS);
        if (j == nt - 1 && un >= 0) {
          // the unit's last S has been read: the next unit's Q goes in now
          if (!write_q(lv + 1)) return;
          q_ready_u = un;
          phase(TR_S_MERGE_LOOP);
        }
      }
      // -------- epilogue: combine the two halves' accumulators with the
      // sink, inverse RoPE, store this warp's columns
      float m_o, l_o;
      const long long tx0 = TRACE ? clock64() : 0;
      {
        float2 *xl = reinterpret_cast<float2 *>(xch);
        xl[warp * 32 + lane] = make_float2(m_used, l);
        if (!pair_sync()) return;
        const float2 o2 = xl[(warp ^ 4) * 32 + lane];
        m_o = o2.x;
        l_o = o2.y;
      }
      if (TRACE) tr[TR_P_ISSUE] += clock64() - tx0;   // the pair exchange
      {
        const uint32_t gl = g + nt - 1;
        if (!twait(bar(bars->pv_done[gl % SP]), (gl / SP) & 1, TR_S_EPI_WAIT)) return;
      }
      if (TRACE && threadIdx.x == 0 && ts[3] == 0) ts[3] = global_ns();
      const long long te0 = TRACE ? clock64() : 0;
      tc_fence_after();
      // weights of accumulator 0 (keys [0, 32) of each tile) and 1
      const float m0 = hf ? m_o : m_used, m1 = hf ? m_used : m_o;
      const float l0 = hf ? l_o : l, l1 = hf ? l : l_o;
      const float mm = fmaxf(m0, m1);
      float w0 = 0.f, w1 = 0.f, inv = 0.f;
      if (mm != -INFINITY) {
        w0 = m0 == -INFINITY ? 0.f : exp2f(m0 - mm);
        w1 = m1 == -INFINITY ? 0.f : exp2f(m1 - mm);
        const float sink2 = live ? p.sink[rh] * kLog2e : 0.f;
        inv = 1.f / (w0 * l0 + w1 * l1 + exp2f(sink2 - mm));
      }
      w0 *= inv;
      w1 *= inv;
#pragma unroll 1
      for (int c0 = col_lo; c0 < col_lo + CH; c0 += 16) {
        uint32_t o0[16], o1[16];
        tmem_ld_32x32b_x16(tmem + lane_base + c0, o0);
        tmem_ld_32x32b_x16(tmem + lane_base + C + c0, o1);
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) v[x] = __uint_as_float(o0[x]) * w0 + __uint_as_float(o1[x]) * w1;
        if (c0 + 16 > C - p.rd) {
#pragma unroll
          for (int x = 0; x < 16; x += 2) {
            const int col = c0 + x;
            if (col >= C - p.rd) {
              const int pi = (col - (C - p.rd)) / 2;
              const float cs = rope_cs[pi], sn = rope_cs[32 + pi];
              const float a = v[x], bb = v[x + 1];
              v[x] = a * cs + bb * sn;
              v[x + 1] = -a * sn + bb * cs;
            }
          }
        }
        if (live) {
          uint4 ww0, ww1;
          ww0.x = pack_bf16x2(v[0], v[1]); ww0.y = pack_bf16x2(v[2], v[3]);
          ww0.z = pack_bf16x2(v[4], v[5]); ww0.w = pack_bf16x2(v[6], v[7]);
          ww1.x = pack_bf16x2(v[8], v[9]); ww1.y = pack_bf16x2(v[10], v[11]);
          ww1.z = pack_bf16x2(v[12], v[13]); ww1.w = pack_bf16x2(v[14], v[15]);
          *reinterpret_cast<uint4 *>(orow + c0) = ww0;
          *reinterpret_cast<uint4 *>(orow + c0 + 8) = ww1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(bars->o_empty));
        mbar_arrive(bar(bars->us_empty[lv & 1]));   // the unit's slot is free again
      }
      if (TRACE) tr[TR_S_EPI] += clock64() - te0;
      if (TRACE && threadIdx.x == 0 && ts[4] == 0) ts[4] = global_ns();
      g += nt;
      ++lv;
    }
    }();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    [&]() {
    float *rope_cs = rope_all + warp * 64;
    const int q4 = warp;                  // TMEM lane quarter
    const int hl = lane & 15, half = lane >> 4;
    const int r = q4 * 16 + hl;           // MMA row
    // row r is head rh of query rg of the unit's group; every row of a warp
    // belongs to query wg of the group (n_h is a multiple of 16 when G > 1)
    const int rg = r / p.n_h, rh = r - rg * p.n_h;
    const int wg = p.G > 1 ? (q4 * 16) / p.n_h : 0;
    const float zs = p.scale * kLog2e;
    const uint32_t lane_S = (uint32_t)(q4 * 32 + 16) << 16;
    const uint32_t lane_O = (uint32_t)(q4 * 32) << 16;
    // Q of a unit into tensor memory (lane-half 1, columns q_col..): thread
    // (hl, half) stores head row r, bf16 dims [half*C/2, (half+1)*C/2), read
    // from global in batches of 16 x 16 B whose loads are all in flight
    uint32_t nq = 0;                      // Q writes so far (q_empty parity)
    auto write_q = [&](int uq) -> bool {
      if (nq > 0 && !twait(bar(bars->q_empty), (nq - 1) & 1, TR_P_QEMPTY)) return false;
      tc_fence_after();
      const Unit xq = unit_of(p, uq);
      const bool live = rg < p.G && xq.qi0 + rg < p.n_q;
      const long long qrow = live ? ((long long)xq.b * p.n_q + xq.qi0 + rg) * p.n_h + rh : 0;
      const uint4 *src = reinterpret_cast<const uint4 *>(
          reinterpret_cast<const __nv_bfloat16 *>(p.q) + qrow * C + half * (C / 2));
      const uint32_t tq = tmem + lane_S + L::q_col;
      // C/16 uint4 (C/4 words) per thread, in batches of 16 uint4 whose loads are all in flight
      constexpr int PER = C / 16, BATCH = PER < 16 ? PER : 16;
#pragma unroll 1
      for (int b0 = 0; b0 < PER; b0 += BATCH) {
        uint4 v[BATCH];
#pragma unroll
        for (int x = 0; x < BATCH; ++x) v[x] = live ? __ldg(src + b0 + x) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int y = 0; y < BATCH / 4; ++y)
          tmem_st_16x32bx2_x16<C / 4>(tq + 4 * (b0 + 4 * y), *reinterpret_cast<const uint32_t(*)[16]>(&v[4 * y]));
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bars->q_full));
      ++nq;
      return true;
    };
    // the next unit of this CTA with key tiles (its Q is written ahead), or -1
    auto next_unit = [&](int u0) -> int {
      for (int uu = u0 + gridDim.x; uu < n_units; uu += gridDim.x) {
        int a0, an;
        const Unit xu = unit_of(p, uu);
        split_range(group_key_set(p, xu.qg), p.nsplit, xu.sp, a0, an);
        if (an > 0) return uu;
      }
      return -1;
    };
    int q_ready_u = -1;                   // unit whose Q is already in tensor memory
    uint32_t g = 0, iq = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      const Unit ux = unit_of(p, u);
      const int bq = ux.bq, sp = ux.sp, b = ux.b, qi = ux.qi0;
      const int t = p.start_pos + qi + wg;   // this warp's query token
      const bool live = rg < p.G && qi + rg < p.n_q;
      const KeySet ks = group_key_set(p, ux.qg);
      int j0, nt;
      split_range(ks, p.nsplit, sp, j0, nt);
      if (nt > 0 && q_ready_u != u) {
        if (!write_q(u)) return;
        q_ready_u = u;
      }
      {
        // pull the next unit's Q rows towards L2 now; they are written to tensor
        // memory after this unit's last S
        const int un = next_unit(u);
        const Unit xn = unit_of(p, un < 0 ? 0 : un);
        if (un >= 0 && rg < p.G && xn.qi0 + rg < p.n_q) {
          const char *nq = reinterpret_cast<const char *>(
              reinterpret_cast<const __nv_bfloat16 *>(p.q) +
              (((long long)xn.b * p.n_q + xn.qi0 + rg) * p.n_h + rh) * C + half * (C / 2));
#pragma unroll
          for (int x = 0; x < C / 128; ++x) asm volatile("prefetch.global.L2 [%0];" ::"l"(nq + 128 * x));
        }
      }
      if (nt == 0 && p.nsplit > 1 && !p.cluster) continue;   // the combine kernel skips empty ranges
      __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) +
                            (live ? (((long long)b * p.n_q + qi + rg) * p.n_h + rh) * C : 0);
      if (nt == 0 && !p.cluster) {
        if (live)
          for (int col = half * (C / 2); col < (half + 1) * (C / 2); col += 8)
            *reinterpret_cast<uint4 *>(orow + col) = make_uint4(0, 0, 0, 0);
        continue;
      }
      // RoPE table of this token (inverse rotation applied in the epilogue)
      __syncwarp();
      if (lane < p.rd / 2) {
        const double two_pi = 6.283185307179586476925286766559;
        double ang = (double)t * freq[lane];
        ang -= two_pi * floor(ang / two_pi);
        float sn, cs;
        sincosf((float)ang, &sn, &cs);
        rope_cs[lane] = cs;
        rope_cs[32 + lane] = sn;
      }
      __syncwarp();
      float m_used = -INFINITY, l = 0.f;
      if (TRACE) { tr[TR_UNITS] += 1; tr[TR_TILES] += nt; }
      for (int j = 0; j < nt; ++j) {
        const uint32_t gj = g + j;
        const int st = gj % SP;
        const uint32_t ph = (gj / SP) & 1;
        if (!twait(bar(bars->s_full[st]), ph, TR_S_SFULL)) return;
        if (TRACE && threadIdx.x == 0 && j == 0 && ts[2] == 0) ts[2] = global_ns();
        tc_fence_after();
        uint32_t sv[32];
        tmem_ld_16x32bx2_x16<32>(tmem + lane_S + L::s_col(st), *reinterpret_cast<uint32_t(*)[16]>(&sv[0]));
        tmem_ld_16x32bx2_x16<32>(tmem + lane_S + L::s_col(st) + 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[16]));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bars->s_empty[st]));
        // validity of the tile's 64 keys: lane l checks keys l and 32+l, shared by ballot
        const int kbase = (j0 + j) * KT + half * 32;
        uint32_t vmask;
        {
          const int k0 = (j0 + j) * KT + lane, k1 = k0 + 32;
          bool v0 = false, v1 = false;
          if (p.G > 1) {
            v0 = k0 < ks.nk && slot_of_token(p, ks, k0, t);
            v1 = k1 < ks.nk && slot_of_token(p, ks, k1, t);
          } else {
            if (k0 < ks.nk) slot_row(p, ks, b, qi, k0, v0);
            if (k1 < ks.nk) slot_row(p, ks, b, qi, k1, v1);
          }
          const uint32_t m0 = __ballot_sync(0xffffffffu, v0), m1 = __ballot_sync(0xffffffffu, v1);
          vmask = half ? m1 : m0;
        }
        float z[32];
        float tmax = -INFINITY;
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          z[x] = ((vmask >> x) & 1u) ? __uint_as_float(sv[x]) * zs : -INFINITY;
          tmax = fmaxf(tmax, z[x]);
        }
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        bool need = false;
        float alpha = 1.f;
        if (j == 0) {
          m_used = (tmax == -INFINITY) ? 0.f : tmax;
        } else if (tmax > m_used + 8.f) {
          need = true;
          alpha = exp2f(m_used - tmax);
          m_used = tmax;
          l *= alpha;
        }
        if (__any_sync(0xffffffffu, need)) {
          // rescale O rows of this warp after the PV of the previous tile lands
          const uint32_t gp = gj - 1;
          if (TRACE) tr[TR_RESCALES] += 1;
          if (!twait(bar(bars->pv_done[gp % SP]), (gp / SP) & 1, TR_S_RESCALE)) return;
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < C / 2; c0 += 16) {
            uint32_t ov[16];
            tmem_ld_16x32bx2_x16<C / 2>(tmem + lane_O + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 16; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
            tmem_st_16x32bx2_x16<C / 2>(tmem + lane_O + c0, ov);
          }
          tmem_st_wait();
        }
        float psum = 0.f;
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float p0 = ex2_approx(z[x] - m_used), p1 = ex2_approx(z[x + 1] - m_used);
          psum += p0 + p1;
          pk[x / 2] = pack_bf16x2(p0, p1);
        }
        l += psum;
        // P buffer `st` is free once the PV of tile gj-3 has completed
        if (!twait(bar(bars->pv_done[st]), ph ^ 1, TR_S_PBUF)) return;
        uint8_t *prow = smem + L::p_off + st * kTileBytes;
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4) {
          const int chunkp = half * 4 + u4;
          *reinterpret_cast<uint4 *>(prow + sw128_off(r, chunkp)) =
              make_uint4(pk[u4 * 4 + 0], pk[u4 * 4 + 1], pk[u4 * 4 + 2], pk[u4 * 4 + 3]);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bars->p_full[st]));
        if (j == nt - 1) {
          // the unit's last S has been read: write the next unit's Q now, so
          // its first S overlaps this unit's last P.V and epilogue
          const int un = next_unit(u);
          if (un >= 0) {
            if (!write_q(un)) return;
            q_ready_u = un;
          }
        }
      }
      // -------- epilogue: normalise, inverse RoPE, store
      if (nt > 0) {
        const uint32_t gl = g + nt - 1;
        if (!twait(bar(bars->pv_done[gl % SP]), (gl / SP) & 1, TR_S_EPI_WAIT)) return;
      }
      if (TRACE && threadIdx.x == 0 && ts[3] == 0) {
        ts[3] = global_ns();
        if (ts[2] == 0) ts[2] = ts[3];
      }
      const long long te0 = TRACE ? clock64() : 0;
      tc_fence_after();
      const float ltot = l + __shfl_xor_sync(0xffffffffu, l, 16);
      if (p.cluster) {
        // (max, sum) of this row into every owner's block, then the shared merge
        if (half == 0) {
          const uint32_t blk = merge_blk(C, p.nsplit);
          const int pitch = merge_pitch(C, p.nsplit);
          for (int j = 0; j < p.nsplit; ++j)
            reinterpret_cast<float2 *>(smem + j * blk + 64u * pitch * 2)[r] =
                make_float2(nt > 0 ? m_used : -INFINITY, nt > 0 ? ltot : 0.f);
        }
        if (!cluster_merge<C>(p, smem, bars, tmem, nt, sp, b, qi, rope_all,
                              TRACE ? &tr[TR_S_MERGE_READY] : nullptr))
          return;
        if (TRACE) tr[TR_S_EPI] += clock64() - te0;
        if (TRACE && threadIdx.x == 0 && ts[4] == 0) ts[4] = global_ns();
        g += nt;
        ++iq;
        continue;
      }
      if (p.nsplit > 1) {
        // unnormalised partial: O rows (fp32), running max (log2 units) and sum
        const long long slot = (long long)bq * p.nsplit + sp;
        float *po = p.part_o + (slot * 64 + r) * C;
        if (half == 0) {
          p.part_ml[(slot * 64 + r) * 2] = m_used;
          p.part_ml[(slot * 64 + r) * 2 + 1] = ltot;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < C / 2; c0 += 16) {
          uint32_t ov[16];
          tmem_ld_16x32bx2_x16<C / 2>(tmem + lane_O + c0, ov);
          tmem_ld_wait();
          float4 *dst = reinterpret_cast<float4 *>(po + half * (C / 2) + c0);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[x] = make_float4(__uint_as_float(ov[4 * x]), __uint_as_float(ov[4 * x + 1]),
                                 __uint_as_float(ov[4 * x + 2]), __uint_as_float(ov[4 * x + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bars->o_empty));
        if (TRACE) tr[TR_S_EPI] += clock64() - te0;
        if (TRACE && threadIdx.x == 0 && ts[4] == 0) ts[4] = global_ns();
        g += nt;
        ++iq;
        continue;
      }
      const float sink2 = live ? p.sink[rh] * kLog2e : 0.f;
      const float inv = 1.f / (ltot + exp2f(sink2 - m_used));
#pragma unroll 1
      for (int c0 = 0; c0 < C / 2; c0 += 16) {
        uint32_t ov[16];
        tmem_ld_16x32bx2_x16<C / 2>(tmem + lane_O + c0, ov);
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) v[x] = __uint_as_float(ov[x]) * inv;
        const int col0 = half * (C / 2) + c0;
        if (col0 + 16 > C - p.rd) {
#pragma unroll
          for (int x = 0; x < 16; x += 2) {
            const int col = col0 + x;
            if (col >= C - p.rd) {
              const int pi = (col - (C - p.rd)) / 2;
              const float cs = rope_cs[pi], sn = rope_cs[32 + pi];
              const float a = v[x], bb = v[x + 1];
              v[x] = a * cs + bb * sn;
              v[x + 1] = -a * sn + bb * cs;
            }
          }
        }
        if (live) {
          uint4 w0, w1;
          w0.x = pack_bf16x2(v[0], v[1]); w0.y = pack_bf16x2(v[2], v[3]);
          w0.z = pack_bf16x2(v[4], v[5]); w0.w = pack_bf16x2(v[6], v[7]);
          w1.x = pack_bf16x2(v[8], v[9]); w1.y = pack_bf16x2(v[10], v[11]);
          w1.z = pack_bf16x2(v[12], v[13]); w1.w = pack_bf16x2(v[14], v[15]);
          *reinterpret_cast<uint4 *>(orow + col0) = w0;
          *reinterpret_cast<uint4 *>(orow + col0 + 8) = w1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bars->o_empty));
      if (TRACE) tr[TR_S_EPI] += clock64() - te0;
      if (TRACE && threadIdx.x == 0 && ts[4] == 0) ts[4] = global_ns();
      g += nt;
      ++iq;
    }
    }();
  }
  if (TRACE) {
    tr[TR_TOTAL] = clock64() - t_start;
    // one thread per role reports: producer thread 0, MMA lane 0, softmax thread 0
    const bool rep = threadIdx.x == PW0 * 32 || threadIdx.x == MMAW * 32 || threadIdx.x == 0;
    if (rep)
      for (int i = 0; i < TR_COUNT; ++i)
        if (tr[i]) atomicAdd(&g_attn_trace[i], tr[i]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (TRACE && threadIdx.x == 0 && ts[4] != 0) {
    ts[5] = global_ns();
    atomicAdd(&g_attn_trace[TR_T_SETUP], ts[1] - ts[0]);
    atomicAdd(&g_attn_trace[TR_T_FIRST_S], ts[2] - ts[1]);
    atomicAdd(&g_attn_trace[TR_T_TILES], ts[3] - ts[2]);
    atomicAdd(&g_attn_trace[TR_T_EPI], ts[4] - ts[3]);
    atomicAdd(&g_attn_trace[TR_T_EXIT], ts[5] - ts[4]);
    atomicMax(&g_attn_trace[TR_T_ENTRY_INV], ~ts[0]);
    atomicMax(&g_attn_trace[TR_T_EXIT_MAX], ts[5]);
    atomicAdd(&g_attn_trace[TR_T_CTAS], 1ull);
  }
  if (threadIdx.x == 0) step_trace_record(p.csa ? ST_ATTEND_CSA : ST_ATTEND_HCA, st_entry, st_ready);
  if (warp == MMAW) tmem_dealloc(tmem, L::tmem_cols);
}

template <int C, int M>
int ensure_attr() {
  static std::atomic<bool> attr_set_dev[kMaxDevices];
  std::atomic<bool> &attr_set = attr_set_dev[device_slot()];
  if (!attr_set) {
    const int smem = (int)Layout<C, M>::bytes;
    cudaError_t e = cudaFuncSetAttribute(attend_tc<C, M, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attend_tc<C, M, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if constexpr (M == 64) {
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(attend_tc<C, M, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(attend_tc<C, M, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    }
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "attend_tc smem attribute: %s", cudaGetErrorString(e));
    attr_set = true;
  }
  return HCA_OK;
}

// How many clusters of `ns` CTAs can be resident at once (0 if unknown).
template <int C>
int max_active_clusters(int ns) {
  static std::atomic<int> cache_dev[kMaxDevices][kMaxClusterSplits + 1];
  if (ns < 1 || ns > kMaxClusterSplits) return 0;
  std::atomic<int> *cache = cache_dev[device_slot()];
  if (cache[ns]) return cache[ns];
  if (ensure_attr<C, 64>()) return 0;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(ns * 64, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout<C>::bytes;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = ns;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attend_tc<C, 64, false, false>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cache[ns] = n;
  return n;
}

template <int C, int M>
int launch_tc(const AttendParams &p, cudaStream_t s) {
  const int n_units = p.B * p.n_qg * p.nsplit;
  const size_t smem = Layout<C, M>::bytes;
  int rc0 = ensure_attr<C, M>();
  if (rc0) return rc0;
  // cluster merge: one unit per CTA, a query's splits form one cluster
  const int grid = p.cluster ? n_units : (n_units < sm_budget(p) ? n_units : sm_budget(p));
  LaunchScope ls_(p.csa ? "attend_csa_tc" : "attend_hca_tc", s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = p.cluster ? p.nsplit : 1;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = p.cluster ? 2 : 1;
  const bool tr = attend_trace_on();
  cudaError_t e;
  if constexpr (M == 128) {
    e = tr ? cudaLaunchKernelEx(&cfg, attend_tc<C, M, true, false>, p, n_units)
           : cudaLaunchKernelEx(&cfg, attend_tc<C, M, false, false>, p, n_units);
  } else {
    e = p.kv_mixed ? (tr ? cudaLaunchKernelEx(&cfg, attend_tc<C, M, true, true>, p, n_units)
                         : cudaLaunchKernelEx(&cfg, attend_tc<C, M, false, true>, p, n_units))
                   : (tr ? cudaLaunchKernelEx(&cfg, attend_tc<C, M, true, false>, p, n_units)
                         : cudaLaunchKernelEx(&cfg, attend_tc<C, M, false, false>, p, n_units));
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(HCA_ERR_CUDA, "attend_tc launch: %s", cudaGetErrorString(e));
  }
  return ls_.done();
}
}  // namespace tc

}  // namespace

namespace {
bool tc_path(const AttendParams &p) {
  return p.dtype == HCA_BF16 && p.n_h <= 64 && (p.c == 128 || p.c == 256 || p.c == 512) && p.rd <= p.c / 2 &&
         p.rd % 2 == 0 && p.rd <= 64;
}
// Splits per query: enough work units to fill the GPU when there are few queries.
int choose_splits_raw(const AttendParams &p) {
  const long long q = (long long)p.B * p.n_q;
  const int sms = sm_budget(p);
  if (q == 0 || q >= sms) return 1;
  // longest key list among the queries (the last one)
  const int t = p.start_pos + p.n_q - 1;
  const int V = (t + 1) / p.m;
  const int nk = (p.w < t + 1 ? p.w : t + 1) + (p.csa ? (p.k < V ? p.k : V) : V);
  const int tiles = (nk + 63) / 64;
  int ns = (int)(sms / q);                // every unit in one wave of persistent CTAs
  if (ns > tiles / 2) ns = tiles / 2;     // keep >= 2 tiles per split
  if (ns > 32) ns = 32;
  return ns < 1 ? 1 : ns;
}
int max_active_clusters_for(const AttendParams &p, int ns) {
  switch (p.c) {
    case 128: return tc::max_active_clusters<128>(ns);
    case 256: return tc::max_active_clusters<256>(ns);
    default: return tc::max_active_clusters<512>(ns);
  }
}
// Split plan: with at most 8 splits per query the splits of a query run as
// one thread-block cluster and merge through distributed shared memory (no
// workspace, no combine launch); the split count is lowered until all the
// clusters are resident at once.  More splits go through the workspace and
// the combine kernel when the caller gave one, else are cut to 8.
struct SplitPlan {
  int ns, cluster;
};
SplitPlan plan_splits(const AttendParams &p, bool have_ws) {
  SplitPlan sp{choose_splits_raw(p), 0};
  if (sp.ns <= 1 || (sp.ns > tc::kMaxClusterSplits && have_ws)) return sp;
  if (sp.ns > tc::kMaxClusterSplits) sp.ns = tc::kMaxClusterSplits;
  {
    const long long q = (long long)p.B * p.n_q;
    int ns = sp.ns;
    while (ns > 1) {
      const int fit = max_active_clusters_for(p, ns);
      if (fit == 0 || fit >= q) break;   // unknown occupancy: keep the split count
      --ns;
    }
    sp.ns = ns;
    sp.cluster = ns > 1;
  }
  return sp;
}
}  // namespace

size_t attend_workspace_bytes(const AttendParams &p) {
  if (!tc_path(p)) return 0;
  const SplitPlan sp = plan_splits(p, true);
  const int ns = sp.ns;
  if (ns <= 1 || sp.cluster) return 0;
  const size_t q = (size_t)p.B * p.n_q * ns * 64;
  return ((q * p.c * 4 + 255) & ~(size_t)255) + ((q * 8 + 255) & ~(size_t)255);
}

int run_attend(const AttendParams &p_in, void *ws, size_t ws_bytes, cudaStream_t s) {
  if (p_in.B * p_in.n_q == 0) return HCA_OK;
  AttendParams p = p_in;
  for (int i = 0; i < 32; ++i)
    p.rope_freq[i] = i < p.rd / 2 ? std::exp2(-2.0 * i / (double)p.rd * std::log2((double)p.theta)) : 0.0;
  p.nsplit = 1;
  p.cluster = 0;
  p.G = 1;
  p.n_qg = p.n_q;
  p.fd_m = make_fastdiv((uint32_t)p.m);
  p.fd_nsplit = make_fastdiv(1);
  p.fd_nqg = make_fastdiv((uint32_t)p.n_qg);
  if (p.kv_mixed && !tc_path(p))
    return fail(HCA_ERR_UNSUPPORTED, "mixed-precision KV rows need the tensor-core path (bf16, n_h <= 64, c in {128, 256, 512})");
  if (tc_path(p)) {
    if (!p.kv_comp) p.cap = 0;   // no visible entries: masked slots then read row 0 of the dummy map
    const SplitPlan sp = plan_splits(p, ws && ws_bytes >= attend_workspace_bytes(p));
    const int ns = sp.ns;
    if (ns == 1 && !p.csa && !p.win_is_ring && p.n_q > 1 && p.n_h % 16 == 0) {
      // G = rows / n_h queries per unit fill the MMA's 128 rows (c = 128,
      // bf16 rows) or 64 rows; kept while the groups still give every CTA of
      // the budget a unit
      for (int rows = (p.c == 128 && !p.kv_mixed) ? 128 : 64; rows >= 64; rows -= 64) {
        const int G = rows / p.n_h, n_qg = (p.n_q + G - 1) / G;
        if (G >= 2 && rows % p.n_h == 0 && (long long)p.B * n_qg >= sm_budget(p)) {
          p.G = G;
          p.n_qg = n_qg;
          break;
        }
      }
    }
    if (sp.cluster) {
      p.nsplit = ns;
      p.cluster = 1;
    } else if (ns > 1 && ws && ws_bytes >= attend_workspace_bytes(p)) {
      p.nsplit = ns;
      const size_t q = (size_t)p.B * p.n_q * ns * 64;
      p.part_o = static_cast<float *>(ws);
      p.part_ml = reinterpret_cast<float *>(static_cast<char *>(ws) + ((q * p.c * 4 + 255) & ~(size_t)255));
    }
    p.fd_nsplit = make_fastdiv((uint32_t)p.nsplit);
    p.fd_nqg = make_fastdiv((uint32_t)p.n_qg);
    const bool m128 = p.G * p.n_h == 128;
    int rc;
    switch (p.c) {
      case 128: rc = m128 ? tc::launch_tc<128, 128>(p, s) : tc::launch_tc<128, 64>(p, s); break;
      case 256: rc = tc::launch_tc<256, 64>(p, s); break;
      default: rc = tc::launch_tc<512, 64>(p, s); break;
    }
    if (rc || p.nsplit == 1 || p.cluster) return rc;
    return HCA_LAUNCH("attend_combine", s, attend_combine<__nv_bfloat16><<<dim3(p.B * p.n_q, (p.n_h + 3) / 4), 128, 0, s>>>(p));
  }
  dim3 grid(p.B * p.n_q, (p.n_h + kSimtWarps - 1) / kSimtWarps);
  const size_t smem = (size_t)kSimtKT * p.c * sizeof(float);
  LaunchScope ls_(p.csa ? "attend_csa_simt" : "attend_hca_simt", s);
  if (p.dtype == HCA_F32) attend_simt<float><<<grid, kSimtWarps * 32, smem, s>>>(p);
  else attend_simt<__nv_bfloat16><<<grid, kSimtWarps * 32, smem, s>>>(p);
  return ls_.done();
}

int step_trace_set_attend(void *buf, unsigned long long cap) { return step_trace_set_here(buf, cap); }

}  // namespace hca

extern "C" int hca_trace_attend(int enable, unsigned long long *host_counters, int n) {
  using namespace hca;
  if (host_counters && n > 0) {
    unsigned long long buf[32];
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyFromSymbol(buf, tc::g_attn_trace, sizeof buf) != cudaSuccess)
      return fail(HCA_ERR_CUDA, "trace read failed");
    for (int i = 0; i < n && i < 32; ++i) host_counters[i] = buf[i];
  }
  if (enable >= 0) {
    const unsigned long long zero[32] = {0};
    if (cudaMemcpyToSymbol(tc::g_attn_trace, zero, sizeof zero) != cudaSuccess)
      return fail(HCA_ERR_CUDA, "trace reset failed");
    tc::g_trace_on = enable != 0;
  }
  return HCA_OK;
}
