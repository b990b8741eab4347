// rvq_norms.cu -- codeword norms ||C_l[k]||^2, the bf16 tensor-core operand copy and the
// per-level statistics that bound the error of bf16 distances.  Runs once per fixed
// codebook set (LongCat-2.5 blog, "Offline Visual Preprocessing": the tokenizer is fixed).
// HBM-bound: one read of [L,K,D] (+ one bf16 write when the codebooks are fp32).
#include <cuda_bf16.h>

#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {

// Non-negative floats order like their bit patterns, so atomicMax on the bits is a float max.
__device__ __forceinline__ void atomic_max_nonneg(float *addr, float v) {
  atomicMax(reinterpret_cast<unsigned int *>(addr), __float_as_uint(v));
}

// One warp per codeword.  Lanes stride over D in chunks of 4 elements.
template <bool CB_BF16>
__global__ void __launch_bounds__(256) norms_kernel(const void *__restrict__ cb, int L, int K, int D,
                                                    float *__restrict__ norms, float *__restrict__ stats,
                                                    __nv_bfloat16 *__restrict__ cb_op) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t total = static_cast<int64_t>(L) * K;
  if (w >= total) return;
  const int l = static_cast<int>(w / K);
  double s_c = 0.0, s_q = 0.0, s_e = 0.0;  // ||c||^2, ||bf16(c)||^2, ||c - bf16(c)||^2
  if constexpr (CB_BF16) {
    const __nv_bfloat16 *row = static_cast<const __nv_bfloat16 *>(cb) + w * D;
    for (int i = lane * 4; i < D; i += 128) {
      uint2 raw = *reinterpret_cast<const uint2 *>(row + i);
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float2 f = __bfloat1622float2(h[j]);
        s_c += static_cast<double>(f.x) * f.x + static_cast<double>(f.y) * f.y;
      }
    }
    s_q = s_c;
  } else {
    const float *row = static_cast<const float *>(cb) + w * D;
    __nv_bfloat16 *orow = cb_op + w * D;
    for (int i = lane * 4; i < D; i += 128) {
      float4 f = *reinterpret_cast<const float4 *>(row + i);
      __nv_bfloat162 a = __floats2bfloat162_rn(f.x, f.y);
      __nv_bfloat162 b = __floats2bfloat162_rn(f.z, f.w);
      float2 qa = __bfloat1622float2(a), qb = __bfloat1622float2(b);
      s_c += static_cast<double>(f.x) * f.x + static_cast<double>(f.y) * f.y + static_cast<double>(f.z) * f.z +
             static_cast<double>(f.w) * f.w;
      s_q += static_cast<double>(qa.x) * qa.x + static_cast<double>(qa.y) * qa.y +
             static_cast<double>(qb.x) * qb.x + static_cast<double>(qb.y) * qb.y;
      double e0 = static_cast<double>(f.x) - qa.x, e1 = static_cast<double>(f.y) - qa.y;
      double e2 = static_cast<double>(f.z) - qb.x, e3 = static_cast<double>(f.w) - qb.y;
      s_e += e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
      uint2 packed;
      packed.x = *reinterpret_cast<uint32_t *>(&a);
      packed.y = *reinterpret_cast<uint32_t *>(&b);
      *reinterpret_cast<uint2 *>(orow + i) = packed;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s_c += __shfl_xor_sync(0xffffffffu, s_c, o);
    s_q += __shfl_xor_sync(0xffffffffu, s_q, o);
    s_e += __shfl_xor_sync(0xffffffffu, s_e, o);
  }
  if (lane == 0) {
    norms[w] = __double2float_rn(s_c);
    float *st = stats + static_cast<int64_t>(l) * RVQ_LEVEL_STATS;
    atomic_max_nonneg(st + 0, __double2float_ru(sqrt(s_c)));
    atomic_max_nonneg(st + 1, __double2float_ru(sqrt(s_e)));
    atomic_max_nonneg(st + 2, __double2float_ru(sqrt(s_q)));
    atomic_max_nonneg(st + 3, __double2float_ru(s_c));
  }
}

}  // namespace rvq

extern "C" int rvq_build_norms(const void *codebooks, int cb_dtype, int L, int K, int D, float *norms,
                               float *level_stats, void *cb_operand, void *stream) {
  using namespace rvq;
  if (!codebooks || !norms || !level_stats) return RVQ_ERR_ARG;
  if (cb_dtype != RVQ_F32 && cb_dtype != RVQ_BF16) return RVQ_ERR_ARG;
  if (L < 1 || K < 1 || D < 1) return RVQ_ERR_ARG;
  if (L > 64 || D < 16 || D > 8192 || D % 16 != 0) return RVQ_ERR_UNSUPPORTED;
  if (cb_dtype == RVQ_F32 && !cb_operand) return RVQ_ERR_ARG;
  if (!aligned16(codebooks) || !aligned16(norms) || (cb_operand && !aligned16(cb_operand)))
    return RVQ_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(level_stats, 0, sizeof(float) * RVQ_LEVEL_STATS * L, s) != cudaSuccess)
    return RVQ_ERR_CUDA;
  const int64_t warps = static_cast<int64_t>(L) * K;
  const int64_t blocks = (warps + 7) / 8;
  if (blocks > 0x7FFFFFFFLL) return RVQ_ERR_UNSUPPORTED;
  if (cb_dtype == RVQ_BF16)
    norms_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, s>>>(codebooks, L, K, D, norms, level_stats,
                                                                      nullptr);
  else
    norms_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        codebooks, L, K, D, norms, level_stats, static_cast<__nv_bfloat16 *>(cb_operand));
  note_launch();
  return check_launch();
}
