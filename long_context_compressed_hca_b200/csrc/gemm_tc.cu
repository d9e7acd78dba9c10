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

}  // namespace

int launch_gemm_tc(const void *A, long long lda, const void *Bm, long long ldb, void *C, long long ldc,
                   hca_dtype cdt, int M, int N, int K, float alpha, cudaStream_t s) {
  // full tiles of B rows and 16-byte row pitches for TMA; otherwise the caller uses the SIMT GEMM
  if (M < BM || N < BN || K < BK || (lda * 2) % 16 || (ldb * 2) % 16 ||
      (reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(Bm) & 15))
    return HCA_ERR_UNSUPPORTED;
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
