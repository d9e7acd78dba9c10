// index_tc.cu -- lightning-indexer scores on the 5th-generation tensor cores.
//
// I[t,s] = sum_h w[t,h] ReLU(q^I[t,h] . K^I[s])   (juejin "DeepSeek-V4 技术报告简要解读"
// §2.3.1(b) Eq.(16); 1zeryu "DeepSeek-V4：算法架构", Indexer einsum + ReLU·w sum).
//
// Computed as a swapped GEMM D[s, (t,h)] = K^I[s, :] . q^I[(t,h), :] with the
// entries on the MMA's M = 128 rows and a block of queries x indexer heads on
// N (16..256), K = c_I = 64 (one 128-byte swizzle block).  The ReLU, the
// weighted head sum and the fp8 row scale run in the epilogue straight out
// of TMEM: thread = entry, so each score row segment is written coalesced.
//
// Roles: warp 0 streams key tiles (TMA 2-D, 128B swizzle; fp8 tiles go to a
// staging buffer and warps 10-13 widen them to bf16), warp 1 issues the MMAs
// into a double-buffered TMEM accumulator, warps 2-9 run the epilogue.
#include "common.cuh"
#include "internal.h"

namespace hca {
namespace {

constexpr int kRowsA = 128;                   // entries per tile (MMA M)
constexpr uint32_t kTileA = kRowsA * 128;     // 16 KB bf16 key tile
constexpr uint32_t kStageF8 = kRowsA * 64;    // 8 KB fp8 staging tile
constexpr int kEpiWarps = 8;

struct TcIdxArgs {
  int B, n_q, start_pos, m, n_hI, cap, QB;    // QB queries per block
  int tiles_per_unit, units_per_qb, n_qb;
  const float *wI, *KI_scale;
  float *scores;
  long long score_stride;
  int *status;
  int round_bf16;
};

template <int N, bool FP8, int S>
struct TcIdxLayout {
  static constexpr uint32_t a_off = 0;
  static constexpr uint32_t b_off = S * kTileA;
  static constexpr uint32_t st_off = b_off + ((N * 128 + 1023) / 1024) * 1024;
  static constexpr uint32_t w_off = st_off + (FP8 ? S * kStageF8 : 0);
  static constexpr uint32_t bar_off = w_off + 1024;                 // w: up to 256 floats
  static constexpr uint32_t bytes = bar_off + 512 + 1024;
  static constexpr uint32_t tmem_cols = 2 * N < 32 ? 32 : 2 * N;
  static constexpr int threads = (2 + kEpiWarps + (FP8 ? 4 : 0)) * 32;
};

template <int N, bool FP8, int S>
__global__ void __launch_bounds__(TcIdxLayout<N, FP8, S>::threads, 1)
index_scores_tc(TcIdxArgs p, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ) {
  using L = TcIdxLayout<N, FP8, S>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::bar_off);
  // bars: [0,S) a_full, [S,2S) a_empty, [2S,3S) st_full, [3S,4S) st_empty, 4S b_full,
  //       4S+1..+2 acc_full, 4S+3..+4 acc_empty
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::bar_off + 8 * (4 * S + 8));
  float *wsm = reinterpret_cast<float *>(smem + L::w_off);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int a_full = 0, a_empty = S, st_full = 2 * S, st_empty = 3 * S, b_full = 4 * S, acc_full = 4 * S + 1,
            acc_empty = 4 * S + 3;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned long long st_entry = global_ns();
  // work unit: (sequence, query block, tile range)
  int u = blockIdx.x;
  const int nunits_per_b = p.n_qb * p.units_per_qb;
  const int b = u / nunits_per_b;
  u %= nunits_per_b;
  const int qb = p.n_qb - 1 - u / p.units_per_qb;        // largest blocks first
  const int chunk = u % p.units_per_qb;
  const int q0 = qb * p.QB;
  const int nq = min(p.QB, p.n_q - q0);
  const int v_last = (p.start_pos + q0 + nq) / p.m;      // entries visible to the last query
  const int e_begin = chunk * p.tiles_per_unit * kRowsA;
  const int e_end = min(v_last, e_begin + p.tiles_per_unit * kRowsA);
  const int nt = e_end > e_begin ? (e_end - e_begin + kRowsA - 1) / kRowsA : 0;
  if (nt == 0) return;   // uniform for the whole block, before any barrier use

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(bar(a_full + i), FP8 ? 128 : 1);
      mbar_init(bar(a_empty + i), 1);
      mbar_init(bar(st_full + i), 1);
      mbar_init(bar(st_empty + i), 128);
    }
    mbar_init(bar(b_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(acc_full + i), 1);
      mbar_init(bar(acc_empty + i), kEpiWarps);
    }
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long key_row0 = (long long)b * p.cap + e_begin;
  pdl_trigger();   // the selection may start its prologue
  pdl_wait();      // keys and queries of the previous launch are complete
  const unsigned long long st_ready = global_ns();

  if (warp == 0) {
    // ------------------------------------------------ loads
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmQ);
      mbar_arrive_expect_tx(bar(b_full), N * 128);
      tma_load_2d(sbase + L::b_off, &tmQ, 0, (b * p.n_q + q0) * p.n_hI, bar(b_full));
      for (int j = 0; j < nt; ++j) {
        const int st = j % S;
        const uint32_t ph = (j / S) & 1;
        if (FP8) {
          if (!mbar_wait(bar(st_empty + st), ph ^ 1, p.status)) break;
          mbar_arrive_expect_tx(bar(st_full + st), kStageF8);
          tma_load_2d(sbase + L::st_off + st * kStageF8, &tmK, 0, (int)(key_row0 + j * kRowsA), bar(st_full + st));
        } else {
          if (!mbar_wait(bar(a_empty + st), ph ^ 1, p.status)) break;
          mbar_arrive_expect_tx(bar(a_full + st), kTileA);
          tma_load_2d(sbase + L::a_off + st * kTileA, &tmK, 0, (int)(key_row0 + j * kRowsA), bar(a_full + st));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, N, 0, 0);
      bool ok = mbar_wait(bar(b_full), 0, p.status);
      for (int j = 0; j < nt && ok; ++j) {
        const int st = j % S, ab = j & 1;
        if (!mbar_wait(bar(a_full + st), (j / S) & 1, p.status) ||
            !mbar_wait(bar(acc_empty + ab), ((j >> 1) & 1) ^ 1, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = sbase + L::a_off + st * kTileA, bq = sbase + L::b_off;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem + ab * N, sdesc_sw128(a + kk * 32, 16, 1024), sdesc_sw128(bq + kk * 32, 16, 1024), IDESC,
                    kk > 0 ? 1u : 0u);
        umma_commit(bar(a_empty + st));
        umma_commit(bar(acc_full + ab));
      }
      // drain: the last commit's barrier completes when every MMA is done
      if (ok) mbar_wait(bar(acc_full + ((nt - 1) & 1)), ((nt - 1) >> 1) & 1, p.status);
    }
    __syncwarp();
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------ epilogue: ReLU, weighted head sum, store
    const int ew = warp - 2;
    const int quarter = warp & 3;                       // TMEM lane quarter of this warp
    const int group = ew >> 2;                          // which half of the query block
    const int et = threadIdx.x - 64;
    for (int i = et; i < nq * p.n_hI; i += kEpiWarps * 32)
      wsm[i] = p.wI[((long long)b * p.n_q + q0) * p.n_hI + i];
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    // D column = query * 8 + head (n_hI == 8): each 8-column chunk is one query
    [&]() {
      for (int j = 0; j < nt; ++j) {
        const int ab = j & 1;
        if (!mbar_wait(bar(acc_full + ab), (j >> 1) & 1, p.status)) return;
        tc_fence_after();
        const int e = e_begin + j * kRowsA + quarter * 32 + lane;
        float kscale = 1.f;
        if (FP8 && e < e_end) kscale = p.KI_scale[(long long)b * p.cap + e];
        const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + ab * N + group * (N / 2);
#pragma unroll
        for (int c0 = 0; c0 < N / 2; c0 += 8) {
          uint32_t r[8];
          tmem_ld_32x32b_x8(tbase + c0, r);
          tmem_ld_wait();
          const int jq = (group * (N / 2) + c0) >> 3;
          if (jq < nq) {
            float sacc = 0.f;
#pragma unroll
            for (int x = 0; x < 8; ++x) sacc += wsm[jq * 8 + x] * fmaxf(__uint_as_float(r[x]), 0.f);
            const int t = p.start_pos + q0 + jq;
            float v = sacc * kscale;
            if (p.round_bf16) v = __bfloat162float(__float2bfloat16_rn(v));
            if (e < e_end && e < (t + 1) / p.m)
              p.scores[((long long)b * p.n_q + q0 + jq) * p.score_stride + e] = v;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(acc_empty + ab));
      }
    }();
  } else if (FP8) {
    // ------------------------------------------------ fp8 -> bf16 widening (warps 10-13)
    const int ct = threadIdx.x - (2 + kEpiWarps) * 32;   // 0..127 = row of the tile
    [&]() {
      for (int j = 0; j < nt; ++j) {
        const int st = j % S;
        const uint32_t ph = (j / S) & 1;
        if (!mbar_wait(bar(st_full + st), ph, p.status)) return;
        if (!mbar_wait(bar(a_empty + st), ph ^ 1, p.status)) return;
        const uint8_t *src = smem + L::st_off + st * kStageF8 + ct * 64;
        uint8_t *dst = smem + L::a_off + st * kTileA;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = *reinterpret_cast<const uint4 *>(src + q * 16);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // two e4m3 pairs -> two bf16 pairs (exact: e4m3 fits in bf16)
            __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w4[i] & 0xFFFF), __NV_E4M3);
            __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w4[i] >> 16), __NV_E4M3);
            const float2 f01 = __half22float2(__half2(h01));
            const float2 f23 = __half22float2(__half2(h23));
            o[2 * i] = pack_bf16x2(f01.x, f01.y);
            o[2 * i + 1] = pack_bf16x2(f23.x, f23.y);
          }
          *reinterpret_cast<uint4 *>(dst + sw128_off(ct, 2 * q)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4 *>(dst + sw128_off(ct, 2 * q + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
        fence_proxy_async();
        mbar_arrive(bar(st_empty + st));
        mbar_arrive(bar(a_full + st));
      }
    }();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) step_trace_record(ST_INDEX, st_entry, st_ready);
  if (warp == 1) tmem_dealloc(tmem, L::tmem_cols);
}

template <int N, bool FP8, int S>
int launch_tc_t(const IndexParams &p, int QB, int tiles_per_unit, int units_per_qb, cudaStream_t s) {
  using L = TcIdxLayout<N, FP8, S>;
  static std::atomic<bool> attr_dev[kMaxDevices];
  std::atomic<bool> &attr = attr_dev[device_slot()];
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(index_scores_tc<N, FP8, S>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return fail(HCA_ERR_CUDA, "index_tc smem attribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  CUtensorMap tmK, tmQ;
  int rc;
  if (FP8)
    rc = encode_tmap_2d(&tmK, p.KI, CU_TENSOR_MAP_DATA_TYPE_UINT8, 64, (uint64_t)p.B * p.cap, 64, 64, kRowsA,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    rc = encode_tmap_2d(&tmK, p.KI, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, (uint64_t)p.B * p.cap, 128, 64, kRowsA,
                        CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  rc = encode_tmap_2d(&tmQ, p.qI, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, (uint64_t)p.B * p.n_q * p.n_hI, 128, 64,
                      N, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  TcIdxArgs a{};
  a.B = p.B; a.n_q = p.n_q; a.start_pos = p.start_pos; a.m = p.m; a.n_hI = p.n_hI; a.cap = p.cap; a.QB = QB;
  a.tiles_per_unit = tiles_per_unit; a.units_per_qb = units_per_qb; a.n_qb = (p.n_q + QB - 1) / QB;
  a.wI = p.wI; a.KI_scale = p.KI_scale; a.scores = p.scores; a.score_stride = p.score_stride; a.status = p.status;
  a.round_bf16 = p.round_bf16;
  const long long grid = (long long)p.B * a.n_qb * units_per_qb;
  LaunchScope ls_(FP8 ? "index_scores_tc_fp8" : "index_scores_tc", s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(L::threads, 1, 1);
  cfg.dynamicSmemBytes = L::bytes;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, index_scores_tc<N, FP8, S>, a, tmK, tmQ);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(HCA_ERR_CUDA, "index_scores_tc launch: %s", cudaGetErrorString(e));
  }
  return ls_.done();
}

}  // namespace

int launch_index_scores_tc(const IndexParams &p, cudaStream_t s) {
  const bool fp8 = p.key_dtype == HCA_FP8E4M3;
  if (p.q_dtype != HCA_BF16 || !(fp8 || p.key_dtype == HCA_BF16) || p.c_I != 64 || p.n_hI != 8)
    return HCA_ERR_UNSUPPORTED;
  const int Vmax = (p.start_pos + p.n_q) / p.m;
  if (Vmax == 0) return HCA_OK;
  if ((reinterpret_cast<uintptr_t>(p.KI) | reinterpret_cast<uintptr_t>(p.qI)) & 15) return HCA_ERR_UNSUPPORTED;
  if (p.n_q >= 16) {
    // prefill: 16 queries x 8 heads per block, every tile of the block's range
    const int tiles = (Vmax + kRowsA - 1) / kRowsA;
    return fp8 ? launch_tc_t<128, true, 4>(p, 16, tiles, 1, s) : launch_tc_t<128, false, 4>(p, 16, tiles, 1, s);
  }
  // decode / short: 2 queries per block, the entry range cut into units so that
  // every SM streams keys
  const int n_qb = (p.n_q + 1) / 2;
  const int tiles = (Vmax + kRowsA - 1) / kRowsA;
  // two resident blocks per SM.  With many query pairs, four waves of them: units
  // small enough for the grid to balance over the SMs that another stream's
  // kernels leave free (32 sequences in the two-layer decode step, the other
  // layer's attention beside it: one wave 112 us per step, four waves 106 us).
  // With few (4 sequences at 1M entries) one wave, which measured faster there.
  const long long want = ((long long)p.B * n_qb >= 16 ? 8LL : 2LL) * num_sms();
  int units = (int)(want / ((long long)p.B * n_qb));
  if (units > tiles) units = tiles;
  if (units < 1) units = 1;
  const int tpu = (tiles + units - 1) / units;
  units = (tiles + tpu - 1) / tpu;
  return fp8 ? launch_tc_t<16, true, 6>(p, 2, tpu, units, s) : launch_tc_t<16, false, 6>(p, 2, tpu, units, s);
}

int step_trace_set_index_tc(void *buf, unsigned long long cap) { return step_trace_set_here(buf, cap); }

}  // namespace hca
