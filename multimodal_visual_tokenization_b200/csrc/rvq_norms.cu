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

// One warp per codeword, eight codewords per block.  Each lane accumulates its strided share
// of the row in fp32 (at most D/32 terms), lane sums are combined in fp64; the per-level maxima
// are reduced in the block first so only one atomic per block and statistic reaches L2.
template <bool CB_BF16>
__global__ void __launch_bounds__(256) norms_kernel(const void *__restrict__ cb, int L, int K, int D,
                                                    float *__restrict__ norms, float *__restrict__ stats,
                                                    __nv_bfloat16 *__restrict__ cb_op) {
  __shared__ float wmax[8][RVQ_LEVEL_STATS];
  __shared__ int wlev[8];
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  const int64_t total = static_cast<int64_t>(L) * K;
  const bool live = w < total;
  float s_c = 0.f, s_q = 0.f, s_e = 0.f;  // lane shares of ||c||^2, ||bf16(c)||^2, ||c - bf16(c)||^2
  if (live) {
    if constexpr (CB_BF16) {
      const __nv_bfloat16 *row = static_cast<const __nv_bfloat16 *>(cb) + w * D;
      for (int i0 = lane * 8; i0 < D; i0 += 1024) {
        uint4 raw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // four 16-byte loads in flight per lane
          const int i = i0 + u * 256;
          raw[u] = (i + 8 <= D) ? __ldg(reinterpret_cast<const uint4 *>(row + i)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t wd[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wd[k]));
            s_c = fmaf(f.x, f.x, s_c);
            s_c = fmaf(f.y, f.y, s_c);
          }
        }
      }
      s_q = s_c;
    } else {
      const float *row = static_cast<const float *>(cb) + w * D;
      __nv_bfloat16 *orow = cb_op + w * D;
      for (int i0 = lane * 4; i0 < D; i0 += 512) {
        float4 f[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // four 16-byte loads in flight per lane
          const int i = i0 + u * 128;
          f[u] = i < D ? __ldg(reinterpret_cast<const float4 *>(row + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * 128;
          if (i >= D) break;
          const __nv_bfloat162 a = __floats2bfloat162_rn(f[u].x, f[u].y);
          const __nv_bfloat162 b = __floats2bfloat162_rn(f[u].z, f[u].w);
          const float2 qa = __bfloat1622float2(a), qb = __bfloat1622float2(b);
          const float v[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
          const float q[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            s_c = fmaf(v[k], v[k], s_c);
            s_q = fmaf(q[k], q[k], s_q);
            const float e = v[k] - q[k];  // exact: the bf16 rounding error of an fp32 value
            s_e = fmaf(e, e, s_e);
          }
          uint2 packed;
          packed.x = *reinterpret_cast<const uint32_t *>(&a);
          packed.y = *reinterpret_cast<const uint32_t *>(&b);
          *reinterpret_cast<uint2 *>(orow + i) = packed;
        }
      }
    }
  }
  double dc = s_c, dq = s_q, de = s_e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dc += __shfl_xor_sync(0xffffffffu, dc, o);
    dq += __shfl_xor_sync(0xffffffffu, dq, o);
    de += __shfl_xor_sync(0xffffffffu, de, o);
  }
  if (lane == 0) {
    wlev[warp] = live ? static_cast<int>(w / K) : -1;
    if (live) {
      norms[w] = __double2float_rn(dc);
      wmax[warp][0] = __double2float_ru(sqrt(dc));
      wmax[warp][1] = __double2float_ru(sqrt(de));
      wmax[warp][2] = __double2float_ru(sqrt(dq));
      wmax[warp][3] = __double2float_ru(dc);
    }
  }
  __syncthreads();
  // thread (warp j, stat k) publishes warp j's maximum unless an earlier warp of the block is
  // on the same level, in which case that warp's thread folds it in
  if (threadIdx.x < 8 * RVQ_LEVEL_STATS) {
    const int j = threadIdx.x / RVQ_LEVEL_STATS, k = threadIdx.x % RVQ_LEVEL_STATS;
    const int lev = wlev[j];
    if (lev >= 0 && (j == 0 || wlev[j - 1] != lev)) {
      float m = wmax[j][k];
      for (int jj = j + 1; jj < 8 && wlev[jj] == lev; ++jj) m = fmaxf(m, wmax[jj][k]);
      atomic_max_nonneg(stats + static_cast<int64_t>(lev) * RVQ_LEVEL_STATS + k, m);
    }
  }
}

}  // namespace rvq

extern "C" int rvq_build_norms(const void *codebooks, int cb_dtype, int L, int K, int D, float *norms,
                               float *level_stats, void *cb_operand, void *stream) {
  RVQ_ENTRY("rvq_build_norms");
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
  cudaError_t e;
  if (cb_dtype == RVQ_BF16)
    e = launch_pdl(norms_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, codebooks, L, K, D,
                   norms, level_stats, static_cast<__nv_bfloat16 *>(nullptr));
  else
    e = launch_pdl(norms_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, codebooks, L, K, D,
                   norms, level_stats, static_cast<__nv_bfloat16 *>(cb_operand));
  note_launch();
  return e == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}
