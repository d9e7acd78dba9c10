// kv_mixed.cu -- KV rows in the mixed-precision cache format.
//
// juejin "DeepSeek-V4 技术报告简要解读" §2.3.4: the KV cache keeps the RoPE
// dims in BF16 and the other dims in FP8, which nearly halves it.  1zeryu
// "DeepSeek-V4：算法架构", "Q, K, V 映射与位置编码注入" and the Compressor:
// after RoPE, the non-RoPE dims of every KV row are quantised to FP8 in blocks
// of 64 channels.
//
// One record per row (hca_kv_mixed_row_bytes): the c - rd e4m3 codes, the rd
// bf16 RoPE channels, one fp32 scale per 64 codes, zero padding to 16 bytes.
// Both kernels are HBM-bound streams: one warp per row, 16 channels per lane
// (c <= 512), 16- and 32-byte accesses; the four lanes of a 64-channel block
// take its amax with two shuffles.
#include "common.cuh"
#include "internal.h"

namespace hca {

namespace {

constexpr int kKvWarps = 8;

__device__ __forceinline__ void load16(const float *p, float *v) {
  const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 a = __ldg(q + i);
    v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
  }
}
__device__ __forceinline__ void load16(const __nv_bfloat16 *p, float *v) {
  const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 a = __ldg(q + i);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
      v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
}
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(a));
  const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(b));
  return lo | (hi << 16);
}
__device__ __forceinline__ void store_bf16x16(unsigned char *dst, const float *v) {
  uint4 *d = reinterpret_cast<uint4 *>(dst);
  d[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
  d[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                    pack_bf16x2(v[14], v[15]));
}

// x: [rows, c] of T; out: rows records of `rec` bytes.
template <typename T>
__global__ void __launch_bounds__(kKvWarps * 32) kv_quant_mixed_kernel(const T *__restrict__ x, long long rows,
                                                                         int c, int rd, unsigned char *__restrict__ out,
                                                                         int rec, long long per_seq, long long seq_rows) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int nq = c - rd, ncl = nq / 16, L = c / 16;
  const int payload = nq + 2 * rd + nq / 16;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
    float v[16];
    if (lane < L) {
      load16(x + r * c + 16 * lane, v);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.f;
    }
    unsigned char *rp = out + ((r / per_seq) * seq_rows + r % per_seq) * rec;
    // the amax of this lane's block (lanes 4b .. 4b+3 hold block b)
    float amax = 0.f;
    if (lane < ncl) {
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    if (lane < ncl) {
      const float scale = __fdiv_rn(amax, 448.0f);
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float q = scale > 0.f ? __fdiv_rn(v[i], scale) : 0.f;
        uint32_t b = (uint32_t)__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
        if ((b & 0x7Fu) == 0u) b = 0u;   // zero is stored as +0
        w[i >> 2] |= b << (8 * (i & 3));
      }
      *reinterpret_cast<uint4 *>(rp + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
      if ((lane & 3) == 0) *reinterpret_cast<float *>(rp + nq + 2 * rd + 4 * (lane >> 2)) = scale;
    } else if (lane < L) {
      store_bf16x16(rp + nq + 32 * (lane - ncl), v);
    }
    for (int b = payload + 4 * lane; b < rec; b += 128) *reinterpret_cast<uint32_t *>(rp + b) = 0u;
  }
}

// in: rows records; out: [rows, c] bf16.
__global__ void __launch_bounds__(kKvWarps * 32) kv_dequant_mixed_kernel(const unsigned char *__restrict__ in,
                                                                           long long rows, int c, int rd,
                                                                           __nv_bfloat16 *__restrict__ out, int rec) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int nq = c - rd, ncl = nq / 16, L = c / 16;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
    const unsigned char *rp = in + r * rec;
    unsigned char *op = reinterpret_cast<unsigned char *>(out + r * c);
    if (lane < ncl) {
      const uint4 cw = __ldg(reinterpret_cast<const uint4 *>(rp + 16 * lane));
      const float scale = __ldg(reinterpret_cast<const float *>(rp + nq + 2 * rd + 4 * (lane >> 2)));
      const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const __nv_fp8_storage_t b = (__nv_fp8_storage_t)((w[i >> 2] >> (8 * (i & 3))) & 0xFFu);
        const __half h = __half(__nv_cvt_fp8_to_halfraw(b, __NV_E4M3));
        v[i] = __half2float(h) * scale;
      }
      store_bf16x16(op + 32 * lane, v);
    } else if (lane < L) {
      const uint4 *s = reinterpret_cast<const uint4 *>(rp + nq + 32 * (lane - ncl));
      uint4 *d = reinterpret_cast<uint4 *>(op + 2 * nq + 32 * (lane - ncl));
      d[0] = __ldg(s);
      d[1] = __ldg(s + 1);
    }
  }
}

int kv_grid(long long rows) {
  const long long blocks = (rows + kKvWarps - 1) / kKvWarps;
  const long long cap = (long long)num_sms() * 16;
  return (int)(blocks < cap ? blocks : cap);
}

}  // namespace

size_t kv_mixed_row_bytes(int c, int rd) {
  if (c < 16 || c > 512 || rd < 0 || rd > c || rd % 16 != 0 || (c - rd) % 64 != 0) return 0;
  const size_t payload = (size_t)(c - rd) + 2 * (size_t)rd + (size_t)(c - rd) / 16;
  return (payload + 15) & ~(size_t)15;
}

int launch_kv_quant_mixed(const void *x, hca_dtype dt, long long rows, int c, int rd, void *out, cudaStream_t s,
                          long long per_seq, long long seq_rows) {
  if (rows == 0) return HCA_OK;
  if (per_seq <= 0) { per_seq = rows; seq_rows = 0; }
  const int rec = (int)kv_mixed_row_bytes(c, rd);
  unsigned char *o = static_cast<unsigned char *>(out);
  if (dt == HCA_F32)
    return HCA_LAUNCH("kv_quant_mixed", s,
                      kv_quant_mixed_kernel<float><<<kv_grid(rows), kKvWarps * 32, 0, s>>>(
                          static_cast<const float *>(x), rows, c, rd, o, rec, per_seq, seq_rows));
  return HCA_LAUNCH("kv_quant_mixed", s,
                    kv_quant_mixed_kernel<__nv_bfloat16><<<kv_grid(rows), kKvWarps * 32, 0, s>>>(
                        static_cast<const __nv_bfloat16 *>(x), rows, c, rd, o, rec, per_seq, seq_rows));
}

int launch_kv_dequant_mixed(const void *in, long long rows, int c, int rd, void *out, cudaStream_t s) {
  if (rows == 0) return HCA_OK;
  const int rec = (int)kv_mixed_row_bytes(c, rd);
  return HCA_LAUNCH("kv_dequant_mixed", s,
                    kv_dequant_mixed_kernel<<<kv_grid(rows), kKvWarps * 32, 0, s>>>(
                        static_cast<const unsigned char *>(in), rows, c, rd, static_cast<__nv_bfloat16 *>(out),
                        rec));
}

}  // namespace hca
