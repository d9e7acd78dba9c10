// gemm_glue.cu -- projections and row-wise glue of the layer path.
//
// The projections of juejin "DeepSeek-V4 技术报告简要解读" Eq.(9)-(10), (13)-(15),
// (18), (20)-(21) and the window-KV projection (1zeryu "DeepSeek-V4：算法架构",
// "Q, K, V 映射与位置编码注入") are plain GEMMs C = A B^T with weights stored
// [d_out, d_in].  The row op fuses RMSNorm (optionally per head), partial RoPE,
// scaling and the storage conversion that follow them.
#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {

// ------------------------------------------------------------------ SIMT GEMM
constexpr int BM = 64, BN = 64, BK = 16;

template <typename Tab, typename Tc>
__global__ void __launch_bounds__(256) gemm_simt(const Tab *A, long long lda, const Tab *B, long long ldb,
                                                 Tc *C, long long ldc, int M, int N, int K, float alpha) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int e = threadIdx.x; e < BM * BK; e += 256) {
      const int r = e / BK, kk = e % BK;
      const int gm = m0 + r, gk = k0 + kk;
      As[kk][r] = (gm < M && gk < K) ? Elt<Tab>::load(A + (long long)gm * lda + gk) : 0.f;
      const int gn = n0 + r;
      Bs[kk][r] = (gn < N && gk < K) ? Elt<Tab>::load(B + (long long)gn * ldb + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn < N) Elt<Tc>::store(C + (long long)gm * ldc + gn, acc[i][j] * alpha);
    }
  }
}

// ------------------------------------------------------- few output columns
// C[M, N] for N <= 32 (the head-weight projection W_w, N = n_hI): one CTA per
// row of A, its threads striding over K (coalesced); each thread keeps N
// partial sums, reduced across the warps at the end (a fixed order).  A's row
// is read once, B (N x K) stays in L1/L2 for every row.
constexpr int kNarrowThreads = 256;
template <typename Tab, typename Tc, int NT>
__global__ void __launch_bounds__(kNarrowThreads) gemm_narrow(const Tab *A, long long lda, const Tab *B,
                                                              long long ldb, Tc *C, long long ldc, int M, int N,
                                                              int K, float alpha) {
  __shared__ float part[kNarrowThreads / 32][NT];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long m = blockIdx.x;
  const Tab *a = A + m * lda;
  float acc[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) acc[j] = 0.f;
#pragma unroll 4
  for (int k = threadIdx.x; k < K; k += kNarrowThreads) {
    const float av = Elt<Tab>::load(a + k);
#pragma unroll
    for (int j = 0; j < NT; ++j)
      if (j < N) acc[j] += av * Elt<Tab>::load(B + (long long)j * ldb + k);
  }
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const float v = warp_sum(acc[j]);
    if (lane == 0) part[warp][j] = v;
  }
  __syncthreads();
  if (threadIdx.x < N) {
    float v = 0.f;
    for (int w = 0; w < kNarrowThreads / 32; ++w) v += part[w][threadIdx.x];
    Elt<Tc>::store(C + m * ldc + threadIdx.x, v * alpha);
  }
}

template <typename Tab, typename Tc>
int launch_narrow(const Tab *A, long long lda, const Tab *B, long long ldb, Tc *C, long long ldc, int M, int N, int K,
                  float alpha, cudaStream_t s) {
  const dim3 grid((unsigned)M);
  LaunchScope ls_("gemm_narrow", s);
  if (N <= 8)
    gemm_narrow<Tab, Tc, 8><<<grid, kNarrowThreads, 0, s>>>(A, lda, B, ldb, C, ldc, M, N, K, alpha);
  else if (N <= 16)
    gemm_narrow<Tab, Tc, 16><<<grid, kNarrowThreads, 0, s>>>(A, lda, B, ldb, C, ldc, M, N, K, alpha);
  else
    gemm_narrow<Tab, Tc, 32><<<grid, kNarrowThreads, 0, s>>>(A, lda, B, ldb, C, ldc, M, N, K, alpha);
  return ls_.done();
}

// ------------------------------------------------------------------ row op
// One warp per row: optional RMS normalisation, gamma, scale, RoPE of the
// last rd columns (interleaved pairs) and conversion.  cols % 4 == 0 rows
// use 16-byte loads; a RoPE pair always sits inside one thread's 4 columns.
constexpr int kRowWarps = 8;

template <typename Tout>
__device__ __forceinline__ void store_cols4(Tout *dst, const float (&v)[4]);
template <>
__device__ __forceinline__ void store_cols4<float>(float *dst, const float (&v)[4]) {
  *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store_cols4<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&v)[4]) {
  *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

template <typename Tout, bool VEC>
__global__ void __launch_bounds__(kRowWarps * 32) row_op_kernel(RowOpParams p) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (row >= p.rows) return;
  const float *in = p.in + row * p.in_stride;
  Tout *out = reinterpret_cast<Tout *>(p.out) + row * p.out_stride;
  float r = p.scale;
  if (p.norm) {
    float ss = 0.f;
    if (VEC) {
      for (int c = 4 * lane; c < p.cols; c += 128) {
        const float4 v = *reinterpret_cast<const float4 *>(in + c);
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
      }
    } else {
      for (int c = lane; c < p.cols; c += 32) ss += in[c] * in[c];
    }
    ss = warp_sum(ss);
    r *= rsqrtf(ss / (float)p.cols + p.eps);
  }
  const long long pos = p.pos_base + (p.pos0 + row / p.rows_per_pos) % p.pos_mod;
  const int c_rope = p.rd > 0 ? p.cols - p.rd : p.cols;
  if (VEC) {
    for (int c = 4 * lane; c < p.cols; c += 128) {
      const float4 x = *reinterpret_cast<const float4 *>(in + c);
      float v[4] = {x.x * r, x.y * r, x.z * r, x.w * r};
      if (p.gamma) {
        const float4 g = *reinterpret_cast<const float4 *>(p.gamma + c);
        v[0] *= g.x; v[1] *= g.y; v[2] *= g.z; v[3] *= g.w;
      }
      if (c >= c_rope) {
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
          float s, cs;
          rope_sincos_tab(p.rope_freq, pos, (c + j - c_rope) / 2, p.rd, p.theta, &s, &cs);
          const float a = v[j], b = v[j + 1];
          v[j] = a * cs - b * s;
          v[j + 1] = a * s + b * cs;
        }
      }
      store_cols4<Tout>(out + c, v);
    }
  } else {
    for (int c = 2 * lane; c < p.cols; c += 64) {
      float a = in[c] * r * (p.gamma ? p.gamma[c] : 1.f);
      float b = in[c + 1] * r * (p.gamma ? p.gamma[c + 1] : 1.f);
      if (c >= c_rope) {
        float s, cs;
        rope_sincos_tab(p.rope_freq, pos, (c - c_rope) / 2, p.rd, p.theta, &s, &cs);
        const float a2 = a * cs - b * s, b2 = a * s + b * cs;
        a = a2; b = b2;
      }
      Elt<Tout>::store(out + c, a);
      Elt<Tout>::store(out + c + 1, b);
    }
  }
}

}  // namespace

int launch_gemm(hca_dtype ab, const void *A, long long lda, const void *Bm, long long ldb, void *C,
                long long ldc, hca_dtype cdt, int M, int N, int K, float alpha, cudaStream_t s) {
  if (M == 0 || N == 0) return HCA_OK;
  if (ab == HCA_BF16) {
    const int rc = launch_gemm_tc(A, lda, Bm, ldb, C, ldc, cdt, M, N, K, alpha, s);
    if (rc != HCA_ERR_UNSUPPORTED) return rc;
  }
  if (N <= 32) {
    if (ab == HCA_F32)
      return cdt == HCA_F32 ? launch_narrow((const float *)A, lda, (const float *)Bm, ldb, (float *)C, ldc, M, N, K,
                                            alpha, s)
                            : launch_narrow((const float *)A, lda, (const float *)Bm, ldb, (__nv_bfloat16 *)C, ldc,
                                            M, N, K, alpha, s);
    return cdt == HCA_F32 ? launch_narrow((const __nv_bfloat16 *)A, lda, (const __nv_bfloat16 *)Bm, ldb, (float *)C,
                                          ldc, M, N, K, alpha, s)
                          : launch_narrow((const __nv_bfloat16 *)A, lda, (const __nv_bfloat16 *)Bm, ldb,
                                          (__nv_bfloat16 *)C, ldc, M, N, K, alpha, s);
  }
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  LaunchScope ls_("gemm_simt", s);
  if (ab == HCA_F32) {
    if (cdt == HCA_F32)
      gemm_simt<float, float><<<grid, 256, 0, s>>>((const float *)A, lda, (const float *)Bm, ldb, (float *)C, ldc, M, N, K, alpha);
    else
      gemm_simt<float, __nv_bfloat16><<<grid, 256, 0, s>>>((const float *)A, lda, (const float *)Bm, ldb, (__nv_bfloat16 *)C, ldc, M, N, K, alpha);
  } else {
    if (cdt == HCA_F32)
      gemm_simt<__nv_bfloat16, float><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)A, lda, (const __nv_bfloat16 *)Bm, ldb, (float *)C, ldc, M, N, K, alpha);
    else
      gemm_simt<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)A, lda, (const __nv_bfloat16 *)Bm, ldb, (__nv_bfloat16 *)C, ldc, M, N, K, alpha);
  }
  return ls_.done();
}

int launch_row_op(const RowOpParams &p0, cudaStream_t s) {
  if (p0.rows == 0) return HCA_OK;
  RowOpParams p = p0;
  fill_rope_freq(p.rope_freq, p.rd, p.theta);
  const bool vec = p.cols % 4 == 0 && p.in_stride % 4 == 0 && p.out_stride % 4 == 0 &&
                   (reinterpret_cast<uintptr_t>(p.in) & 15) == 0 && (reinterpret_cast<uintptr_t>(p.out) & 15) == 0 &&
                   (!p.gamma || (reinterpret_cast<uintptr_t>(p.gamma) & 15) == 0);
  const unsigned grid = (unsigned)((p.rows + kRowWarps - 1) / kRowWarps);
  LaunchScope ls_("row_op", s);
  if (p.out_dtype == HCA_F32) {
    if (vec) row_op_kernel<float, true><<<grid, kRowWarps * 32, 0, s>>>(p);
    else row_op_kernel<float, false><<<grid, kRowWarps * 32, 0, s>>>(p);
  } else {
    if (vec) row_op_kernel<__nv_bfloat16, true><<<grid, kRowWarps * 32, 0, s>>>(p);
    else row_op_kernel<__nv_bfloat16, false><<<grid, kRowWarps * 32, 0, s>>>(p);
  }
  return ls_.done();
}

}  // namespace hca
