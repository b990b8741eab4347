// rvq_decode.cu -- gather-sum decode recon[n] = sum_l C_l[ids[n,l]] (LongCat-2.5 blog,
// Figure 1: discrete token sequences are turned back into features for the visual
// de-tokenizer).  ids are read and recon is written once; every (token, level) gathers one
// codeword row, so N*L*D*s bytes of codeword rows cross from L2 to the SMs (16 GiB for 2^20 tokens
// x 8 levels x 1024 bf16 columns, against 4.6 GB of HBM traffic).
//
// Schedule: the feature axis is cut into slices of 32 x (16-byte load) columns and the grid runs
// slice-major (blockIdx.y = slice), so while one slice is being produced only L*K*slice codebook
// elements are live and stay resident in L2; recon is written with streaming stores.  Gathers of
// all levels of a row are in flight at once per warp, and the next row's ids are fetched meanwhile.
// When a slice's live codebook columns would exceed 64 MiB, two or four rows share a warp and the
// slice narrows to a half or a quarter (fp32 codebooks of 4 x 65536 codewords at D = 256: 0.55 vs
// 0.83 ms); rvq_decode_slice_plan reports the choice.
//
// Measured bound (2^20 tokens, 8 levels, [8,16384,1024] bf16): the L2 -> SM delivery of the gathered
// rows, ~10 TB/s for 512-byte row pieces.  A gather-only copy of this kernel takes about as long as
// the whole decode, the recon write alone 0.70 ms; 128- and 256-column slices, a per-lane cp.async
// ring of 3-8 rows per warp and mixed-precision bf16 adds were no faster.
#include <cuda_bf16.h>

#include <algorithm>

#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {

constexpr int kDecodeWarps = 8;
// resident decode_fixed_kernel blocks per SM; measured on detok: 6 -> 2.93 ms, 4 -> 1.80, 3 -> 1.75, 2 -> 1.95
constexpr int kDecodeBlocksPerSm = 3;
constexpr int kDecodeLevelGroup = 8;  // gathers of one row issued together before they are summed
constexpr int kDecodeRows = 1;  // rows per warp in the runtime-level kernel: their gathers are in flight together

// VEC consecutive elements of one codeword row, widened to fp32.
template <bool CB_BF16, int VEC>
struct Gather;

template <>
struct Gather<true, 8> {  // 16-byte load of 8 bf16
  uint4 raw;
  __device__ __forceinline__ void load(const void *cb, int64_t off) {
    raw = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(cb) + off));
  }
  __device__ __forceinline__ void zero() { raw = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void add_to(float *acc) const {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
      acc[2 * k] += f.x;
      acc[2 * k + 1] += f.y;
    }
  }
};

template <>
struct Gather<true, 4> {  // 8-byte load of 4 bf16 (D not a multiple of 8)
  uint2 raw;
  __device__ __forceinline__ void load(const void *cb, int64_t off) {
    raw = __ldg(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(cb) + off));
  }
  __device__ __forceinline__ void zero() { raw = make_uint2(0, 0); }
  __device__ __forceinline__ void add_to(float *acc) const {
    const uint32_t w[2] = {raw.x, raw.y};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
      acc[2 * k] += f.x;
      acc[2 * k + 1] += f.y;
    }
  }
};

template <>
struct Gather<false, 4> {  // 16-byte load of 4 fp32
  float4 raw;
  __device__ __forceinline__ void load(const void *cb, int64_t off) {
    raw = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(cb) + off));
  }
  __device__ __forceinline__ void zero() { raw = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void add_to(float *acc) const {
    acc[0] += raw.x;
    acc[1] += raw.y;
    acc[2] += raw.z;
    acc[3] += raw.w;
  }
};

// One warp per R rows and a slice of 32*VEC columns; lane = VEC consecutive columns.  The gathers of
// eight levels of all R rows are issued back to back with no branch between them (an out-of-range
// id or a lane past D reads a clamped, valid address and is masked afterwards), then each row is
// summed in ascending level order.
template <bool CB_BF16, int VEC, int R>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(const int32_t *__restrict__ ids, int64_t N,
                                                                  int L, const void *__restrict__ cb, int K,
                                                                  int D, float *__restrict__ recon,
                                                                  int32_t *status) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t n0 = (static_cast<int64_t>(blockIdx.x) * kDecodeWarps + (threadIdx.x >> 5)) * R;
  if (n0 >= N) return;  // whole warp
  const int col = blockIdx.y * (32 * VEC) + lane * VEC;
  const bool active = col < D;
  const int colc = active ? col : 0;
  int id_lo[R], id_hi[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t n = n0 + r < N ? n0 + r : N - 1;  // rows past N repeat the last row, never stored
    id_lo[r] = lane < L ? __ldg(ids + n * L + lane) : 0;
    id_hi[r] = lane + 32 < L ? __ldg(ids + n * L + 32 + lane) : 0;
  }
  float acc[R][VEC];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc[r][k] = 0.f;
  bool bad = false;
  for (int l0 = 0; l0 < L; l0 += kDecodeLevelGroup) {
    Gather<CB_BF16, VEC> g[R][kDecodeLevelGroup];
    bool use[R][kDecodeLevelGroup];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int src = l0 < 32 ? id_lo[r] : id_hi[r];
#pragma unroll
      for (int j = 0; j < kDecodeLevelGroup; ++j) {
        const int l = l0 + j;
        const int id = __shfl_sync(0xffffffffu, src, l & 31);
        const bool lv = l < L;
        const bool ok = lv && static_cast<unsigned>(id) < static_cast<unsigned>(K);
        bad |= lv && !ok && n0 + r < N;
        use[r][j] = ok;
        const int lc = lv ? l : L - 1;
        g[r][j].load(cb, (static_cast<int64_t>(lc) * K + (ok ? id : 0)) * D + colc);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < kDecodeLevelGroup; ++j)
        if (use[r][j]) g[r][j].add_to(acc[r]);
  }
  if (active) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (n0 + r >= N) break;
      float4 *dst = reinterpret_cast<float4 *>(recon + (n0 + r) * D + col);
#pragma unroll
      for (int k = 0; k < VEC; k += 4)
        __stcs(dst + k / 4, make_float4(acc[r][k], acc[r][k + 1], acc[r][k + 2], acc[r][k + 3]));
    }
  }
  if (bad && lane == 0 && blockIdx.y == 0) set_status(status, RVQ_ERR_ID_RANGE);
}

// The same with the number of levels known at compile time (LC <= 16): a warp walks rows of one
// slice with all LC gathers of a row in flight at once, and fetches the next rows' ids while the
// current row's gathers are outstanding, so every L2 round trip a warp waits for carries a full row
// of gathers.  RPW rows share a warp (32 / RPW lanes per row), which narrows the slice to
// 32 / RPW * VEC columns: the launch picks RPW so that the slice's live codebook columns (L * K *
// slice * element size bytes) stay within kDecodeLiveBytes of L2.  Three blocks per SM leave each
// thread enough registers to keep all LC gathers of a row live without spilling.
constexpr int64_t kDecodeLiveBytes = int64_t(64) << 20;

template <bool CB_BF16, int VEC, int LC, int RPW>
__global__ void __launch_bounds__(kDecodeWarps * 32, kDecodeBlocksPerSm) decode_fixed_kernel(const int32_t *__restrict__ ids,
                                                                           int64_t N, const void *__restrict__ cb,
                                                                           int K, int D, float *__restrict__ recon,
                                                                           int32_t *status) {
  constexpr int LPR = 32 / RPW;  // lanes per row
  static_assert(LC <= LPR, "a row's ids are held by the lanes of its own group");
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int grp = lane / LPR, gl = lane % LPR;
  const unsigned full = 0xffffffffu;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kDecodeWarps * RPW;
  int64_t base = (static_cast<int64_t>(blockIdx.x) * kDecodeWarps + (threadIdx.x >> 5)) * RPW;
  if (base >= N) return;  // whole warp
  const int col = blockIdx.y * (LPR * VEC) + gl * VEC;
  const bool active = col < D;
  const int colc = active ? col : 0;
  int64_t n = base + grp;
  int myid = (gl < LC && n < N) ? __ldg(ids + n * LC + gl) : 0;
  bool bad = false;
  while (true) {
    // with several rows per warp the last rows may lie past N (never stored); one row per warp
    // never walks past N, and a constant keeps that loop free of the predicate
    const bool live = RPW == 1 || n < N;
    Gather<CB_BF16, VEC> g[LC];
    bool use[LC];
#pragma unroll
    for (int l = 0; l < LC; ++l) {
      const int id = __shfl_sync(full, myid, grp * LPR + l);
      const bool in_range = static_cast<unsigned>(id) < static_cast<unsigned>(K);
      bad |= live && !in_range;
      use[l] = live && in_range;
      g[l].load(cb, (static_cast<int64_t>(l) * K + (use[l] ? id : 0)) * D + colc);
    }
    const int64_t nbase = base + step;
    const int64_t nn = nbase + grp;
    const int nextid = (gl < LC && nn < N) ? __ldg(ids + nn * LC + gl) : 0;
    float acc[VEC];
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
#pragma unroll
    for (int l = 0; l < LC; ++l)
      if (use[l]) g[l].add_to(acc);
    if (active && live) {
      float4 *dst = reinterpret_cast<float4 *>(recon + n * D + col);
#pragma unroll
      for (int k = 0; k < VEC; k += 4) __stcs(dst + k / 4, make_float4(acc[k], acc[k + 1], acc[k + 2], acc[k + 3]));
    }
    if (nbase >= N) break;
    base = nbase;
    n = nn;
    myid = nextid;
  }
  if (bad && gl == 0 && blockIdx.y == 0) set_status(status, RVQ_ERR_ID_RANGE);
}

template <bool CB_BF16, int VEC, int LC, int RPW>
cudaError_t launch_fixed(const int32_t *ids, int64_t N, const void *cb, int K, int D, float *recon, int32_t *status,
                         cudaStream_t s) {
  // per slice, enough blocks to fill every SM at the kernel's occupancy; each warp then walks rows
  // with a stride of the slice's rows per sweep
  int sms = 0;
  if (device_sm_count(&sms) != RVQ_OK) return cudaErrorUnknown;
  const int64_t warps = (N + RPW - 1) / RPW;
  const int64_t gx = std::min<int64_t>((warps + kDecodeWarps - 1) / kDecodeWarps,
                                       static_cast<int64_t>(sms) * kDecodeBlocksPerSm);
  const int width = 32 / RPW * VEC;
  const int gy = (D + width - 1) / width;
  if (gx > 0x7FFFFFFFLL || gy > 65535) return cudaErrorInvalidValue;
  return launch_pdl(decode_fixed_kernel<CB_BF16, VEC, LC, RPW>, dim3(static_cast<unsigned>(gx), gy),
                    dim3(kDecodeWarps * 32), 0, s, ids, N, cb, K, D, recon, status);
}

// Rows per warp for a decode of L levels of K codewords of elem_bytes each: the widest slice whose
// live codebook columns fit kDecodeLiveBytes, or the narrowest one whose lane groups still hold a
// row's L ids.
inline int decode_rows_per_warp(int L, int K, int VEC, int elem_bytes) {
  int rpw = 1;
  while (rpw < 4 && L <= 32 / (2 * rpw) &&
         static_cast<int64_t>(L) * K * (32 / rpw * VEC) * elem_bytes > kDecodeLiveBytes)
    rpw *= 2;
  return rpw;
}

template <bool CB_BF16, int VEC, int LC = 1>
cudaError_t dispatch_fixed(int L, int rpw, const int32_t *ids, int64_t N, const void *cb, int K, int D, float *recon,
                           int32_t *status, cudaStream_t s) {
  if constexpr (LC > 16) {
    return cudaErrorInvalidValue;
  } else {
    if (L == LC) {
      if constexpr (LC <= 8)
        if (rpw == 4) return launch_fixed<CB_BF16, VEC, LC, 4>(ids, N, cb, K, D, recon, status, s);
      if (rpw == 2) return launch_fixed<CB_BF16, VEC, LC, 2>(ids, N, cb, K, D, recon, status, s);
      return launch_fixed<CB_BF16, VEC, LC, 1>(ids, N, cb, K, D, recon, status, s);
    }
    return dispatch_fixed<CB_BF16, VEC, LC + 1>(L, rpw, ids, N, cb, K, D, recon, status, s);
  }
}

template <bool CB_BF16, int VEC>
cudaError_t launch_decode_t(const int32_t *ids, int64_t N, int L, const void *cb, int K, int D, float *recon,
                            int32_t *status, cudaStream_t s, dim3 grid) {
  return launch_pdl(decode_kernel<CB_BF16, VEC, kDecodeRows>, grid, dim3(kDecodeWarps * 32), 0, s, ids, N, L, cb, K,
                    D, recon, status);
}

int launch_decode(const int32_t *ids, int64_t N, int L, const void *cb, int cb_dtype, int K, int D, float *recon,
                  int32_t *status, cudaStream_t s) {
  if (N == 0) return RVQ_OK;
  if (L <= 16) {
    cudaError_t e;
    if (cb_dtype == RVQ_BF16) {
      if (D % 8 == 0)
        e = dispatch_fixed<true, 8>(L, decode_rows_per_warp(L, K, 8, 2), ids, N, cb, K, D, recon, status, s);
      else
        e = dispatch_fixed<true, 4>(L, decode_rows_per_warp(L, K, 4, 2), ids, N, cb, K, D, recon, status, s);
    } else {
      e = dispatch_fixed<false, 4>(L, decode_rows_per_warp(L, K, 4, 4), ids, N, cb, K, D, recon, status, s);
    }
    note_launch();
    return e == cudaSuccess ? RVQ_OK : e == cudaErrorInvalidValue ? RVQ_ERR_UNSUPPORTED : RVQ_ERR_CUDA;
  }
  const int vec = (cb_dtype == RVQ_BF16 && D % 8 == 0) ? 8 : 4;
  const int64_t rows_per_block = static_cast<int64_t>(kDecodeWarps) * kDecodeRows;
  const int64_t gx = (N + rows_per_block - 1) / rows_per_block;
  const int gy = (D + 32 * vec - 1) / (32 * vec);
  if (gx > 0x7FFFFFFFLL || gy > 65535) return RVQ_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  cudaError_t e;
  if (cb_dtype == RVQ_BF16) {
    if (vec == 8)
      e = launch_decode_t<true, 8>(ids, N, L, cb, K, D, recon, status, s, grid);
    else
      e = launch_decode_t<true, 4>(ids, N, L, cb, K, D, recon, status, s, grid);
  } else {
    e = launch_decode_t<false, 4>(ids, N, L, cb, K, D, recon, status, s, grid);
  }
  note_launch();
  return e == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}

}  // namespace rvq

extern "C" int rvq_decode_slice_plan(int L, int K, int D, int cb_dtype, int *rows_per_warp, int *slice_cols) {
  using namespace rvq;
  if (!rows_per_warp || !slice_cols) return RVQ_ERR_ARG;
  if (L < 1 || K < 1 || D < 1) return RVQ_ERR_ARG;
  if (cb_dtype != RVQ_F32 && cb_dtype != RVQ_BF16) return RVQ_ERR_ARG;
  if (L > 64 || D < 4 || D % 4 != 0) return RVQ_ERR_UNSUPPORTED;
  const int vec = (cb_dtype == RVQ_BF16 && D % 8 == 0) ? 8 : 4;
  const int elem = cb_dtype == RVQ_BF16 ? 2 : 4;
  // the same choice launch_decode makes: rows per warp for the fixed-level kernel, one row per warp
  // in the generic kernel (more than 16 levels)
  const int rpw = L <= 16 ? decode_rows_per_warp(L, K, vec, elem) : 1;
  *rows_per_warp = rpw;
  *slice_cols = 32 / rpw * vec;
  return RVQ_OK;
}

extern "C" int rvq_decode(const int32_t *ids, int64_t N, int L, const void *codebooks, int cb_dtype, int K, int D,
                          float *recon, int32_t *status, void *stream) {
  RVQ_ENTRY("rvq_decode");
  using namespace rvq;
  if (N < 0 || L < 1 || K < 1 || D < 1) return RVQ_ERR_ARG;
  if (cb_dtype != RVQ_F32 && cb_dtype != RVQ_BF16) return RVQ_ERR_ARG;
  if (L > 64 || D < 4 || D % 4 != 0) return RVQ_ERR_UNSUPPORTED;
  if (N == 0) return RVQ_OK;
  if (!ids || !codebooks || !recon) return RVQ_ERR_ARG;
  if (!aligned16(codebooks) || !aligned16(recon) || (reinterpret_cast<uintptr_t>(ids) & 3u)) return RVQ_ERR_ARG;
  return launch_decode(ids, N, L, codebooks, cb_dtype, K, D, recon, status, static_cast<cudaStream_t>(stream));
}
