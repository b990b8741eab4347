// rvq_decode.cu -- gather-sum decode recon[n] = sum_l C_l[ids[n,l]] (LongCat-2.5 blog,
// Figure 1: discrete token sequences are turned back into features for the visual
// de-tokenizer).  HBM-bound: ids are read, recon is written once, codebook rows are gathered.
//
// Schedule: the feature axis is cut into 128-column slices and the grid runs slice-major
// (blockIdx.y = slice), so while one slice is being produced only L*K*128 codebook elements
// are live; they stay resident in L2 and DRAM sees each codebook byte about once.  recon is
// written with streaming stores so it does not evict those codebook lines.
#include <cuda_bf16.h>

#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {

constexpr int kDecodeRowsPerWarp = 4;
constexpr int kDecodeWarps = 8;
constexpr int kDecodeSlice = 128;  // columns per slice: 32 lanes x 4

template <bool CB_BF16>
__device__ __forceinline__ float4 load4(const void *cb, int64_t off) {
  if constexpr (CB_BF16) {
    uint2 raw = __ldg(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(cb) + off));
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  } else {
    return __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(cb) + off));
  }
}

template <bool CB_BF16>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(const int32_t *__restrict__ ids, int64_t N,
                                                                  int L, const void *__restrict__ cb, int K,
                                                                  int D, float *__restrict__ recon,
                                                                  int32_t *status) {
  constexpr int R = kDecodeRowsPerWarp;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int col = blockIdx.y * kDecodeSlice + lane * 4;
  const bool active = col < D;
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * kDecodeWarps + warp) * R;

  // lane j holds the ids of levels j and 32+j for each of the warp's rows
  int id_lo[R], id_hi[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t n = row0 + r;
    id_lo[r] = (n < N && lane < L) ? __ldg(ids + n * L + lane) : 0;
    id_hi[r] = (n < N && lane + 32 < L) ? __ldg(ids + n * L + 32 + lane) : 0;
  }
  float4 acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
  bool bad = false;
#pragma unroll 2
  for (int l = 0; l < L; ++l) {
    const int64_t lbase = static_cast<int64_t>(l) * K;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int id = l < 32 ? __shfl_sync(0xffffffffu, id_lo[r], l) : __shfl_sync(0xffffffffu, id_hi[r], l - 32);
      const bool row_ok = row0 + r < N;
      const bool in_range = static_cast<unsigned>(id) < static_cast<unsigned>(K);
      bad |= row_ok && !in_range;
      if (row_ok && in_range && active) {
        float4 c = load4<CB_BF16>(cb, (lbase + id) * D + col);
        acc[r].x += c.x;
        acc[r].y += c.y;
        acc[r].z += c.z;
        acc[r].w += c.w;
      }
    }
  }
  if (active) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t n = row0 + r;
      if (n < N) __stcs(reinterpret_cast<float4 *>(recon + n * D + col), acc[r]);
    }
  }
  if (bad && lane == 0 && blockIdx.y == 0) set_status(status, RVQ_ERR_ID_RANGE);
}

int launch_decode(const int32_t *ids, int64_t N, int L, const void *cb, int cb_dtype, int K, int D, float *recon,
                  int32_t *status, cudaStream_t s) {
  if (N == 0) return RVQ_OK;
  const int64_t rows_per_block = static_cast<int64_t>(kDecodeWarps) * kDecodeRowsPerWarp;
  const int64_t gx = (N + rows_per_block - 1) / rows_per_block;
  const int gy = (D + kDecodeSlice - 1) / kDecodeSlice;
  if (gx > 0x7FFFFFFFLL || gy > 65535) return RVQ_ERR_UNSUPPORTED;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  if (cb_dtype == RVQ_BF16)
    decode_kernel<true><<<grid, kDecodeWarps * 32, 0, s>>>(ids, N, L, cb, K, D, recon, status);
  else
    decode_kernel<false><<<grid, kDecodeWarps * 32, 0, s>>>(ids, N, L, cb, K, D, recon, status);
  note_launch();
  return check_launch();
}

}  // namespace rvq

extern "C" int rvq_decode(const int32_t *ids, int64_t N, int L, const void *codebooks, int cb_dtype, int K, int D,
                          float *recon, int32_t *status, void *stream) {
  using namespace rvq;
  if (N < 0 || L < 1 || K < 1 || D < 1) return RVQ_ERR_ARG;
  if (cb_dtype != RVQ_F32 && cb_dtype != RVQ_BF16) return RVQ_ERR_ARG;
  if (L > 64 || D < 4 || D % 4 != 0) return RVQ_ERR_UNSUPPORTED;
  if (N == 0) return RVQ_OK;
  if (!ids || !codebooks || !recon) return RVQ_ERR_ARG;
  if (!aligned16(codebooks) || !aligned16(recon) || (reinterpret_cast<uintptr_t>(ids) & 3u)) return RVQ_ERR_ARG;
  return launch_decode(ids, N, L, codebooks, cb_dtype, K, D, recon, status, static_cast<cudaStream_t>(stream));
}
