// gather_paths.cu -- how fast can a CTA fill a 128B-swizzled 64-row x 1 KB
// shared-memory tile (the attention key tile)?  Four ways, no compute:
//   mode 0: TMA 2-D tiled boxes (64 rows x 64 columns, 8 per tile)
//   mode 1: TMA tile::gather4 (4 random rows x 64 columns, 128 per tile)
//   mode 2: cp.async 16 B from 8 warps, random rows, addresses resolved first,
//           stage mbarrier armed to complete when the copies land
//   mode 3: ld.global 16 B + st.shared from 8 warps
// Each CTA streams 200 tiles through 3 stages.
// Build: nvcc -O3 -gencode arch=compute_100a,code=sm_100a -o gather_paths gather_paths.cu
// Run:   ./gather_paths <rows of 1 KB> <mode> <ctas> [issuing lanes for mode 1]
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cstdio>
#include <cstdlib>
#include <vector>

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t c) { asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(c)); }
__device__ __forceinline__ void expect_tx(uint32_t bar, uint32_t b) {
  asm volatile("{.reg .b64 s; mbarrier.arrive.expect_tx.shared::cta.b64 s, [%0], %1;}" ::"r"(bar), "r"(b) : "memory");
}
__device__ __forceinline__ bool try_wait(uint32_t bar, uint32_t par) {
  uint32_t ok;
  asm volatile("{.reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0,1,0,p;}"
               : "=r"(ok) : "r"(bar), "r"(par), "r"(100000u) : "memory");
  return ok;
}
__device__ __forceinline__ unsigned long long gns() { unsigned long long t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t par) {
  const unsigned long long t0 = gns();
  for (uint32_t i = 0;; ++i) {
    if (try_wait(bar, par)) return true;
    if ((i & 255u) == 0 && gns() - t0 > 2000000000ull) return false;
  }
}
__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap *m, int x, int y, uint32_t bar) {
  asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
               ::"r"(dst), "l"(m), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void g4(uint32_t dst, const CUtensorMap *m, int x, int y0, int y1, int y2, int y3, uint32_t bar) {
  asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, %6}], [%7];"
               ::"r"(dst), "l"(m), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(bar) : "memory");
}

// mode 0: tiled boxes of 64 rows x 64 cols (8 KB) ; mode 1: gather4 (4 rows x 64 cols)
// stage = 64 rows x 512 cols (64 KB): 8 tiled ops or 128 gather4 ops
template <int S>
__global__ void bench(const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmG, int mode,
                      int iters, int nrows, int *err, int lanes_issue, const void *gbuf) {
  extern __shared__ __align__(1024) uint8_t sm[];
  uint8_t *base = (uint8_t *)(((uintptr_t)sm + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[S];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) for (int i = 0; i < S; ++i) mbar_init(smem_u32(&full[i]), mode >= 2 ? 256 : 1);
  asm volatile("fence.mbarrier_init.release.cluster;");
  __syncthreads();
  if (mode >= 2) {
    if (warp == 0) return;
    const int t = threadIdx.x - 32;          // 0..255
    const int chunk = t & 63, r0 = t >> 6;   // 64 chunks of 16 B per row, 4 rows per pass
    for (int it = 0; it < iters; ++it) {
      const int st = it % S;
      if (it >= S && !wait(smem_u32(&full[st]), ((it / S) - 1) & 1)) { if (t == 0) atomicAdd(err, 1); return; }
      const uint32_t dst = smem_u32(base + st * 65536);
      const char *src[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        uint32_t x = blockIdx.x * 7919u + it * 131u + (r0 + 4 * i) * 17u;
        x ^= x >> 16; x *= 0x7feb352du; x ^= x >> 15; x *= 0x846ca68bu; x ^= x >> 16;
        src[i] = (const char *)gbuf + (size_t)(x % (uint32_t)nrows) * 1024 + chunk * 16;
      }
      if (mode == 2) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = r0 + 4 * i;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + (chunk >> 3) * 8192 + r * 128 + (((chunk & 7) ^ (r & 7)) << 4)), "l"(src[i]) : "memory");
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[st])) : "memory");
      } else {
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __ldcg((const uint4 *)src[i]);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = r0 + 4 * i;
          *(uint4 *)(base + st * 65536 + (chunk >> 3) * 8192 + r * 128 + (((chunk & 7) ^ (r & 7)) << 4)) = v[i];
        }
        asm volatile("{.reg .b64 s; mbarrier.arrive.shared::cta.b64 s, [%0];}" ::"r"(smem_u32(&full[st])) : "memory");
      }
    }
    for (int st = 0; st < S && st < iters; ++st) {
      const int last = iters - 1 - ((iters - 1 - st) % S);
      if (last >= 0) wait(smem_u32(&full[st]), (last / S) & 1);
    }
    return;
  }
  if (warp != 0) return;
  uint32_t seed = blockIdx.x * 7919u + 13u;
  for (int it = 0; it < iters; ++it) {
    const int st = it % S;
    if (it >= S) {
      if (!wait(smem_u32(&full[st]), ((it / S) - 1) & 1)) { if (lane == 0) atomicAdd(err, 1); return; }
    }
    __syncwarp();
    const uint32_t dst = smem_u32(base + st * 65536);
    if (lane == 0) expect_tx(smem_u32(&full[st]), 65536);
    __syncwarp();
    if (mode == 0) {
      if (lane < 8) {
        const int row0 = (int)((blockIdx.x * 64ull + it * 64ull * gridDim.x) % (uint64_t)(nrows - 64));
        tma2d(dst + lane * 8192, &tmT, lane * 64, row0, smem_u32(&full[st]));
      }
    } else {
      // 16 groups x 8 column blocks = 128 ops; lanes_issue lanes share them
      for (int op = lane; op < 128; op += lanes_issue) {
        if (lane >= lanes_issue) break;
        const int gi = op & 15, kb = op >> 4;
        uint32_t h = seed + it * 131u + gi * 17u;
        auto rnd = [&](uint32_t x) { x ^= x >> 16; x *= 0x7feb352du; x ^= x >> 15; x *= 0x846ca68bu; x ^= x >> 16; return (int)(x % (uint32_t)nrows); };
        g4(dst + kb * 8192 + gi * 512, &tmG, kb * 64, rnd(h), rnd(h + 1), rnd(h + 2), rnd(h + 3), smem_u32(&full[st]));
      }
    }
  }
  for (int st = 0; st < S && st < iters; ++st) {
    const int last = iters - 1 - ((iters - 1 - st) % S);
    if (last >= 0) wait(smem_u32(&full[st]), (last / S) & 1);
  }
}

int main(int argc, char **argv) {
  const long nrows = atol(argv[1]);       // rows of 512 bf16 (1 KB)
  const int mode = atoi(argv[2]);
  const int ctas = atoi(argv[3]);
  const int lanes = argc > 4 ? atoi(argv[4]) : 32;
  void *buf;
  cudaMalloc(&buf, nrows * 1024);
  cudaMemset(buf, 0, nrows * 1024);
  int *err;
  cudaMalloc(&err, 4);
  cudaMemset(err, 0, 4);
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  cudaDriverEntryPointQueryResult q;
  cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", (void **)&enc, cudaEnableDefault, &q);
  CUtensorMap tmT, tmG;
  cuuint64_t dims[2] = {512, (cuuint64_t)nrows}, str[1] = {1024};
  cuuint32_t boxT[2] = {64, 64}, boxG[2] = {64, 1}, es[2] = {1, 1};
  enc(&tmT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, buf, dims, str, boxT, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  enc(&tmG, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, buf, dims, str, boxG, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  const int S = 3, iters = 200;
  const size_t smem = S * 65536 + 1024;
  cudaFuncSetAttribute(bench<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  for (int rep = 0; rep < 2; ++rep) {
    cudaEventRecord(a);
    bench<3><<<ctas, 288, smem>>>(tmT, tmG, mode, iters, (int)nrows, err, lanes, buf);
    cudaEventRecord(b);
    cudaEventSynchronize(b);
  }
  float ms;
  cudaEventElapsedTime(&ms, a, b);
  int e = 0;
  cudaMemcpy(&e, err, 4, cudaMemcpyDeviceToHost);
  const double bytes = (double)ctas * iters * 65536;
  printf("rows=%ld (%s) mode=%s ctas=%d lanes=%d: %.3f ms  %.1f GB/s total  %.2f GB/s/CTA  err=%d  %s\n", nrows,
         nrows * 1024 > (126l << 20) ? "HBM" : "L2", mode == 0 ? "tiled" : mode == 1 ? "gather4" : mode == 2 ? "cp.async" : "ldg+sts", ctas, lanes, ms, bytes / ms / 1e6,
         bytes / ms / 1e6 / ctas, e, cudaGetErrorString(cudaGetLastError()));
  return 0;
}
