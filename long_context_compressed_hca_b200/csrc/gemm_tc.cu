// gemm_tc.cu -- the layer's projection GEMMs on the tcgen05 tensor cores.
//
// C[M, N] = alpha * A[M, K] . B[N, K]^T with A and B bf16 row-major (K
// contiguous), fp32 accumulation in tensor memory, C fp32 or bf16.  These are
// the projections of the layer glue (juejin "DeepSeek-V4 技术报告简要解读"
// Eq.(9)-(10), (13)-(15), (18), (20)-(21); 1zeryu "DeepSeek-V4：算法架构",
// Q/K/V 映射): compressor C/Z, W_DQ, W_UQ, W_IUQ, window KV.
//
// One 128 x 256 output tile per CTA.  Warp 0 streams 64-wide K slices of A
// (128 rows) and B (256 rows) with 2-D TMA into a 4-stage ring (128B
// swizzle); warp 1 issues tcgen05.mma (M=128, N=256, K=16) into a 256-column
// fp32 accumulator; warps 2-5 read the accumulator back (one TMEM lane
// quarter each), stage their rows in the drained ring and store whole rows.
#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, NST = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;   // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;   // 32 KB
constexpr uint32_t STAGE = A_BYTES + B_BYTES;
constexpr int kThreads = 192;               // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int EPITCH = BN + 4;              // staged row pitch (floats)
constexpr size_t kSmem = NST * STAGE + 256 + 1024;
static_assert(4u * 32u * EPITCH * 4u <= NST * STAGE, "epilogue staging fits in the stage ring");

struct GemmBars {
  uint64_t full[NST], empty[NST], done;
  uint32_t tmem;
};

template <typename TC>
__device__ __forceinline__ void store4(TC *dst, const float *v);
template <>
__device__ __forceinline__ void store4<float>(float *dst, const float *v) {
  *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *dst, const float *v) {
  *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

template <typename TC>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TC *C,
               long long ldc, int M, int N, int K, float alpha, int *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  GemmBars *bars = reinterpret_cast<GemmBars *>(smem + NST * STAGE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int nk = (K + BK - 1) / BK;
  auto bar = [&](uint64_t &b) { return smem_u32(&b); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(bar(bars->full[i]), 1);
      mbar_init(bar(bars->empty[i]), 1);
    }
    mbar_init(bar(bars->done), 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem), BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      for (int k = 0; k < nk; ++k) {
        const int st = k % NST;
        if (k >= NST && !mbar_wait(bar(bars->empty[st]), ((k / NST) - 1) & 1, status)) break;
        mbar_arrive_expect_tx(bar(bars->full[st]), STAGE);
        tma_load_2d(sbase + st * STAGE, &tmA, k * BK, m0, bar(bars->full[st]));
        tma_load_2d(sbase + st * STAGE + A_BYTES, &tmB, k * BK, n0, bar(bars->full[st]));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0, 0);
      for (int k = 0; k < nk; ++k) {
        const int st = k % NST;
        if (!mbar_wait(bar(bars->full[st]), (k / NST) & 1, status)) break;
        tc_fence_after();
        const uint64_t ad = sdesc_sw128(sbase + st * STAGE, 16, 1024);
        const uint64_t bd = sdesc_sw128(sbase + st * STAGE + A_BYTES, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16(tmem, ad + ((kk * 32) >> 4), bd + ((kk * 32) >> 4), IDESC, (k > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(bars->empty[st]));
      }
      umma_commit(bar(bars->done));   // fires once every MMA issued above has completed
    }
    __syncwarp();
  } else {
    // epilogue: warp w reads TMEM lanes 32*(w%4).. (rows of that quarter)
    const int q = warp & 3;
    if (mbar_wait(bar(bars->done), 0, status)) {
      tc_fence_after();
      // the ring is drained: every TMA load was consumed by an MMA that has completed
      float *stg = reinterpret_cast<float *>(smem) + (warp - 2) * 32 * EPITCH;
      const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tq + c0, v);
        tmem_ld_wait();
        float *dst = stg + lane * EPITCH + c0;
#pragma unroll
        for (int x = 0; x < 4; ++x)
          *reinterpret_cast<float4 *>(dst + 4 * x) =
              make_float4(alpha * __uint_as_float(v[4 * x]), alpha * __uint_as_float(v[4 * x + 1]),
                          alpha * __uint_as_float(v[4 * x + 2]), alpha * __uint_as_float(v[4 * x + 3]));
      }
      __syncwarp();
      const bool vec = (ldc % 4) == 0;
      for (int rr = 0; rr < 32; ++rr) {
        const int row = m0 + q * 32 + rr;
        if (row >= M) break;
        const float *src = stg + rr * EPITCH;
        TC *crow = C + (long long)row * ldc;
#pragma unroll
        for (int c = lane * 4; c < BN; c += 128) {
          const int col = n0 + c;
          if (vec && col + 3 < N) {
            store4<TC>(crow + col, src + c);
          } else {
            for (int x = 0; x < 4; ++x)
              if (col + x < N) Elt<TC>::store(crow + col + x, src[c + x]);
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, BN);
}

// Few rows of A (decode: one token per sequence): C = alpha A B^T computed as
// (B A^T)^T, so that 128 rows of B (output features) fill the MMA's M and the
// TN rows of A (tokens, TN = 32 or 64) its N.  The weights stream through an
// 8-stage ring of 64-wide K slices (TMA, 128B swizzle), each with the
// matching slice of A; the accumulator holds TN fp32 columns; warps 2-5 read
// it back (lane = feature) and store token rows with consecutive lanes on
// consecutive features.  With few output tiles the K range is split over the
// S CTAs of a thread-block cluster (gridDim.z = S): each stages its fp32
// partial in its drained ring, and CTA z sums rows [z 128/S, (z+1) 128/S) of
// all S partials through distributed shared memory in the order 0..S-1 (a
// fixed order: no float atomics).  The cluster waits are bounded.
constexpr int SK_NST = 8;
template <int TN>
struct SkinnyLayout {
  static constexpr uint32_t W_BYTES = 128 * BK * 2;   // 16 KB
  static constexpr uint32_t X_BYTES = TN * BK * 2;    // 4 or 8 KB
  static constexpr uint32_t STAGE = W_BYTES + X_BYTES;
  static constexpr size_t smem = SK_NST * STAGE + 256 + 1024;
};

template <typename TC, int TN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_skinny(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TC *C,
               long long ldc, int M, int N, int K, float alpha, int *status) {
  using SL = SkinnyLayout<TN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  struct Bars {
    uint64_t full[SK_NST], empty[SK_NST], done, ready, freed;
    uint32_t tmem;
  };
  Bars *bars = reinterpret_cast<Bars *>(smem + SK_NST * SL::STAGE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128, m0 = blockIdx.y * TN;
  const int S = gridDim.z, z = blockIdx.z;                 // K splits (one cluster)
  const int nk_all = (K + BK - 1) / BK;
  const int kb0 = (int)((long long)z * nk_all / S), kb1 = (int)((long long)(z + 1) * nk_all / S);
  const int nk = kb1 - kb0;
  auto bar = [&](uint64_t &b) { return smem_u32(&b); };
  constexpr uint32_t TCOLS = TN < 32 ? 32 : TN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < SK_NST; ++i) {
      mbar_init(bar(bars->full[i]), 1);
      mbar_init(bar(bars->empty[i]), 1);
    }
    mbar_init(bar(bars->done), 1);
    mbar_init(bar(bars->ready), S);    // one arrival per CTA of the cluster: its partial is staged
    mbar_init(bar(bars->freed), S);    // one arrival per CTA: it has read every partial it needs
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem), TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem;
  // peers arrive on this CTA's barriers only after every CTA initialised its own
  if (S > 1) cluster_sync();

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      for (int k = 0; k < nk; ++k) {
        const int st = k % SK_NST;
        if (k >= SK_NST && !mbar_wait(bar(bars->empty[st]), ((k / SK_NST) - 1) & 1, status)) break;
        mbar_arrive_expect_tx(bar(bars->full[st]), SL::STAGE);
        tma_load_2d(sbase + st * SL::STAGE, &tmB, (kb0 + k) * BK, n0, bar(bars->full[st]));
        tma_load_2d(sbase + st * SL::STAGE + SL::W_BYTES, &tmA, (kb0 + k) * BK, m0, bar(bars->full[st]));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, TN, 0, 0);
      for (int k = 0; k < nk; ++k) {
        const int st = k % SK_NST;
        if (!mbar_wait(bar(bars->full[st]), (k / SK_NST) & 1, status)) break;
        tc_fence_after();
        const uint64_t wd = sdesc_sw128(sbase + st * SL::STAGE, 16, 1024);
        const uint64_t xd = sdesc_sw128(sbase + st * SL::STAGE + SL::W_BYTES, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16(tmem, wd + ((kk * 32) >> 4), xd + ((kk * 32) >> 4), IDESC, (k > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(bars->empty[st]));
      }
      umma_commit(bar(bars->done));
    }
    __syncwarp();
  } else {
    const int q = warp & 3;
    const bool ok = nk > 0 && mbar_wait(bar(bars->done), 0, status);
    if (ok) tc_fence_after();
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    if (S == 1) {
      const int col = n0 + q * 32 + lane;   // this lane's output feature
#pragma unroll 1
      for (int j0 = 0; ok && j0 < TN; j0 += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tq + j0, v);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int row = m0 + j0 + x;
          if (row < M && col < N) Elt<TC>::store(C + (long long)row * ldc + col, alpha * __uint_as_float(v[x]));
        }
      }
    } else {
      // stage this CTA's partial P[j][feature] (fp32) in the drained ring
      float *P = reinterpret_cast<float *>(smem);
      const int r = q * 32 + lane;
#pragma unroll 1
      for (int j0 = 0; j0 < TN; j0 += 16) {
        uint32_t v[16];
        if (ok) {
          tmem_ld_32x32b_x16(tq + j0, v);
          tmem_ld_wait();
        }
#pragma unroll
        for (int x = 0; x < 16; ++x) P[(j0 + x) * 128 + r] = ok ? __uint_as_float(v[x]) : 0.f;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");   // the 4 epilogue warps
      if (warp == 2 && lane == 0)
        for (int j = 0; j < S; ++j) mbar_arrive_cluster(cluster_map(bar(bars->ready), j));
      if (mbar_wait_cluster(bar(bars->ready), 0, status)) {
        // rows [z 128/S, (z+1) 128/S) of the tile, summed over the partials in order
        const int r0 = z * 128 / S, r1 = (z + 1) * 128 / S, nr = r1 - r0;
        const uint32_t pbase = smem_u32(P);
        // kOut outputs per pass, all of their S partial loads in flight before
        // any is added; each sum still runs over CTAs 0..S-1 in order
        constexpr int kOut = 4, kMaxS = 8;
        const int tot = nr * TN;
        for (int it0 = threadIdx.x - 64; it0 < tot; it0 += 128 * kOut) {
          float part[kOut][kMaxS];
#pragma unroll
          for (int o = 0; o < kOut; ++o) {
            const int it = it0 + o * 128;
            const int j = it / nr, rr = r0 + it % nr;
#pragma unroll
            for (int zz = 0; zz < kMaxS; ++zz)
              part[o][zz] = (it < tot && zz < S)
                                ? __uint_as_float(ld_dsmem_u32(cluster_map(pbase + (uint32_t)((j * 128 + rr) * 4), zz)))
                                : 0.f;
          }
#pragma unroll
          for (int o = 0; o < kOut; ++o) {
            const int it = it0 + o * 128;
            if (it >= tot) break;
            const int j = it / nr, rr = r0 + it % nr;
            float acc = 0.f;
#pragma unroll
            for (int zz = 0; zz < kMaxS; ++zz)
              if (zz < S) acc += part[o][zz];
            const int row = m0 + j, col = n0 + rr;
            if (row < M && col < N) Elt<TC>::store(C + (long long)row * ldc + col, alpha * acc);
          }
        }
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (warp == 2 && lane == 0)
        for (int j = 0; j < S; ++j) mbar_arrive_cluster(cluster_map(bar(bars->freed), j));
      // this CTA's partial stays in place until every peer has read it
      mbar_wait_cluster(bar(bars->freed), 0, status);
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TCOLS);
}

template <int TN>
int launch_skinny(const void *A, long long lda, const void *Bm, long long ldb, void *C, long long ldc, hca_dtype cdt,
                  int M, int N, int K, float alpha, cudaStream_t s) {
  using SL = SkinnyLayout<TN>;
  static std::atomic<bool> attr_dev[kMaxDevices];
  std::atomic<bool> &attr = attr_dev[device_slot()];
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_skinny<float, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SL::smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_tc_skinny<__nv_bfloat16, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SL::smem);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "gemm_tc_skinny smem attribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  CUtensorMap tmA, tmB;
  int rc = encode_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, BK,
                          TN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode_tmap_2d(&tmB, Bm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 2, BK,
                        128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  // K splits: enough CTAs for about two per SM, at most 8 (a portable cluster),
  // at least two K slices each
  const long long tiles = (long long)((N + 127) / 128) * ((M + TN - 1) / TN);
  const int nk_all = (K + BK - 1) / BK;
  long long S = 2LL * num_sms() / tiles;
  if (S > 8) S = 8;
  if (S > nk_all / 2) S = nk_all / 2;
  if (S < 1) S = 1;
  LaunchScope ls_("gemm_tc_skinny", s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((N + 127) / 128, (M + TN - 1) / TN, (unsigned)S);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SL::smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = (unsigned)S;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t e =
      cdt == HCA_F32 ? cudaLaunchKernelEx(&cfg, gemm_tc_skinny<float, TN>, tmA, tmB, static_cast<float *>(C), ldc, M, N,
                                          K, alpha, device_status_ptr())
                     : cudaLaunchKernelEx(&cfg, gemm_tc_skinny<__nv_bfloat16, TN>, tmA, tmB,
                                          static_cast<__nv_bfloat16 *>(C), ldc, M, N, K, alpha, device_status_ptr());
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(HCA_ERR_CUDA, "gemm_tc_skinny launch: %s", cudaGetErrorString(e));
  }
  return ls_.done();
}

}  // namespace

int launch_gemm_tc(const void *A, long long lda, const void *Bm, long long ldb, void *C, long long ldc,
                   hca_dtype cdt, int M, int N, int K, float alpha, cudaStream_t s) {
  // 16-byte row pitches and bases for TMA; otherwise the caller uses the SIMT GEMM
  if (K < BK || (lda * 2) % 16 || (ldb * 2) % 16 || (reinterpret_cast<uintptr_t>(A) & 15) ||
      (reinterpret_cast<uintptr_t>(Bm) & 15))
    return HCA_ERR_UNSUPPORTED;
  // few rows (decode tokens) against many output features: the swapped skinny tile
  if (M < BM && M <= 64 && N >= 128)
    return M <= 32 ? launch_skinny<32>(A, lda, Bm, ldb, C, ldc, cdt, M, N, K, alpha, s)
                   : launch_skinny<64>(A, lda, Bm, ldb, C, ldc, cdt, M, N, K, alpha, s);
  // full tiles of B rows
  if (M < BM || N < BN) return HCA_ERR_UNSUPPORTED;
  static std::atomic<bool> attr_dev[kMaxDevices];
  std::atomic<bool> &attr = attr_dev[device_slot()];
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_tc_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmem);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "gemm_tc smem attribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  CUtensorMap tmA, tmB;
  int rc = encode_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, BK,
                          BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode_tmap_2d(&tmB, Bm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 2, BK,
                        BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  const dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  LaunchScope ls_("gemm_tc", s);
  if (cdt == HCA_F32)
    gemm_tc_kernel<float><<<grid, kThreads, kSmem, s>>>(tmA, tmB, static_cast<float *>(C), ldc, M, N, K, alpha,
                                                        device_status_ptr());
  else
    gemm_tc_kernel<__nv_bfloat16><<<grid, kThreads, kSmem, s>>>(tmA, tmB, static_cast<__nv_bfloat16 *>(C), ldc, M,
                                                                N, K, alpha, device_status_ptr());
  return ls_.done();
}

}  // namespace hca
