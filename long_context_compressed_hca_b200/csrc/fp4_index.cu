// fp4_index.cu -- the FP4 indexer path's activations.
//
// juejin "DeepSeek-V4 技术报告简要解读" §4.4: the CSA indexer's QK activations
// are cached, loaded and multiplied in FP4 (E2M1) with fine-grained scales per
// 1 x 32 sub-block, and FP4 -> FP8 dequantisation is lossless (power-of-two
// scales).  1zeryu "DeepSeek-V4：算法架构", Indexer: q^I and the keys are
// rotated by a Hadamard transform before the FP4 simulation.
//
// Each row of 64 values is rotated (fast Walsh-Hadamard butterflies in fp32,
// strides 1, 2, ..., 32, then the exact scale 1/8), cut into blocks of 32 with
// scale 2^(floor(log2 amax) - 2), rounded to E2M1 (nearest, ties to even,
// saturating at 6) and written back as bf16: every E2M1 value times a power of
// two is exactly a bf16 value, so the bf16 tensor-core indexer then computes
// the FP4 path's dot products.  One warp per row, two values per lane
// (elements 2l and 2l+1); the butterflies of stride >= 2 are lane shuffles.
#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {

constexpr int kFp4Warps = 8;

__device__ __forceinline__ void load2(const float *p, float &a, float &b) {
  const float2 v = __ldg(reinterpret_cast<const float2 *>(p));
  a = v.x;
  b = v.y;
}
__device__ __forceinline__ void load2(const __nv_bfloat16 *p, float &a, float &b) {
  const uint32_t w = __ldg(reinterpret_cast<const unsigned int *>(p));
  a = __uint_as_float(w << 16);
  b = __uint_as_float(w & 0xFFFF0000u);
}

// 2^k for k in [-252, 254] as an exact product of two fp32 powers of two.
__device__ __forceinline__ float pow2_hi(int k) { return __uint_as_float((uint32_t)(max(min(k, 127), -126) + 127) << 23); }
__device__ __forceinline__ float times_pow2(float x, int k) {
  const int k1 = max(min(k, 127), -126);
  return x * pow2_hi(k1) * pow2_hi(k - k1);
}
// floor(log2 a) of a finite a > 0 (subnormals included), from the bits.
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t u = __float_as_uint(a);
  const int ex = (int)((u >> 23) & 0xFFu);
  if (ex) return ex - 127;
  return -127 - (__clz(u & 0x7FFFFFu) - 9);   // subnormal: position of the top mantissa bit
}
// Nearest E2M1 value of q (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6), ties to
// the even code, saturating at 6.  Within [0, 2) the values are k/2 with code
// k, in [2, 4) k with code k + 2, in [4, 6] 2k with code k + 4, so rounding k
// to nearest even gives ties to the even code in each range.
__device__ __forceinline__ float e2m1_round(float q) {
  const float a = fminf(fabsf(q), 6.0f);
  float r;
  if (a < 2.0f) r = 0.5f * (float)__float2int_rn(2.0f * a);
  else if (a < 4.0f) r = (float)__float2int_rn(a);
  else r = fminf(2.0f * (float)__float2int_rn(0.5f * a), 6.0f);
  return r == 0.0f ? 0.0f : copysignf(r, q);   // zero is stored as +0
}

// Row r of `rows` sits at row (r / per_seq) * seq_rows + r % per_seq of x and
// out (rows of 64 values; per_seq = rows and seq_rows = 0 for dense rows).
// x and out may be the same buffer: a warp reads its whole row before it
// writes it.
template <typename T>
__global__ void __launch_bounds__(kFp4Warps * 32) fp4_rotate_quant_kernel(const T *x, long long rows,
                                                                            long long per_seq, long long seq_rows,
                                                                            __nv_bfloat16 *out) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long r0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r0 < rows; r0 += nwarps) {
    const long long r = (r0 / per_seq) * seq_rows + r0 % per_seq;
    float a, b;
    load2(x + r * 64 + 2 * lane, a, b);
    // stride 1: the lane's own pair
    {
      const float lo = a, hi = b;
      a = lo + hi;
      b = lo - hi;
    }
    // strides 2 .. 32: partner lane l ^ m holds the other element of each pair
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const float pa = __shfl_xor_sync(0xffffffffu, a, m);
      const float pb = __shfl_xor_sync(0xffffffffu, b, m);
      if (lane & m) {
        a = pa - a;
        b = pb - b;
      } else {
        a = a + pa;
        b = b + pb;
      }
    }
    a *= 0.125f;
    b *= 0.125f;
    // block of 32 = 16 lanes: amax, scale exponent, E2M1, back to values
    float amax = fmaxf(fabsf(a), fabsf(b));
#pragma unroll
    for (int m = 1; m < 16; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const int e = amax > 0.f ? floor_log2(amax) - 2 : 0;
    const float va = times_pow2(e2m1_round(times_pow2(a, -e)), e);
    const float vb = times_pow2(e2m1_round(times_pow2(b, -e)), e);
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(va));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(vb));
    reinterpret_cast<uint32_t *>(out + r * 64)[lane] = lo | (hi << 16);
  }
}

}  // namespace

int launch_fp4_rotate_quant(const void *x, hca_dtype dt, long long rows, void *out, cudaStream_t s,
                            long long per_seq, long long seq_rows) {
  if (rows == 0) return HCA_OK;
  if (per_seq <= 0) { per_seq = rows; seq_rows = 0; }
  const long long blocks = (rows + kFp4Warps - 1) / kFp4Warps;
  const int grid = (int)(blocks < (long long)num_sms() * 16 ? blocks : (long long)num_sms() * 16);
  __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out);
  if (dt == HCA_F32)
    return HCA_LAUNCH("fp4_rotate_quant", s,
                      fp4_rotate_quant_kernel<float><<<grid, kFp4Warps * 32, 0, s>>>(
                          static_cast<const float *>(x), rows, per_seq, seq_rows, o));
  return HCA_LAUNCH("fp4_rotate_quant", s,
                    fp4_rotate_quant_kernel<__nv_bfloat16><<<grid, kFp4Warps * 32, 0, s>>>(
                        static_cast<const __nv_bfloat16 *>(x), rows, per_seq, seq_rows, o));
}

}  // namespace hca
