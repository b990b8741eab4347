// rvq_decode.cu -- gather-sum decode recon[n] = sum_l C_l[ids[n,l]] (LongCat-2.5 blog,
// Figure 1: discrete token sequences are turned back into features for the visual
// de-tokenizer).  HBM-bound: ids are read, recon is written once, codebook rows are gathered.
//
// Schedule: the feature axis is cut into slices of 32 x (16-byte load) columns and the grid runs
// slice-major (blockIdx.y = slice), so while one slice is being produced only L*K*slice codebook
// elements are live; they stay resident in L2 and DRAM sees each codebook byte about once.
// recon is written with streaming stores so it does not evict those codebook lines.  Gathers of
// eight levels are in flight at once per warp to cover L2 latency.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {

constexpr int kDecodeWarps = 8;
#ifndef RVQ_DECODE_BLOCKS_PER_SM
#define RVQ_DECODE_BLOCKS_PER_SM 3  // measured on detok: 6 -> 2.93 ms, 4 -> 1.80, 3 -> 1.75, 2 -> 1.95
#endif
constexpr int kDecodeBlocksPerSm = RVQ_DECODE_BLOCKS_PER_SM;  // resident decode_fixed_kernel blocks per SM
constexpr int kDecodeLevelGroup = 8;  // gathers of one row issued together before they are summed
#ifndef RVQ_DECODE_ROWS
#define RVQ_DECODE_ROWS 1
#endif
constexpr int kDecodeRows = RVQ_DECODE_ROWS;  // rows per warp: their gathers are in flight together
#ifndef RVQ_DECODE_BF16_VEC
#define RVQ_DECODE_BF16_VEC 8
#endif
constexpr int kBf16Vec = RVQ_DECODE_BF16_VEC;  // bf16 elements per lane per gather (8: 256-column slices)

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

// The same with the number of levels known at compile time (LC <= 16): a warp walks rows
// w, w + W, ... of one slice with all LC gathers of a row in flight at once, and fetches the next
// row's ids while the current row's gathers are outstanding, so every L2 round trip a warp
// waits for carries a full row of gathers.  Three blocks per SM leave each thread enough
// registers to keep all LC gathers of a row live without spilling.
template <bool CB_BF16, int VEC, int LC>
__global__ void __launch_bounds__(kDecodeWarps * 32, kDecodeBlocksPerSm) decode_fixed_kernel(const int32_t *__restrict__ ids,
                                                                           int64_t N, const void *__restrict__ cb,
                                                                           int K, int D, float *__restrict__ recon,
                                                                           int32_t *status) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kDecodeWarps;
  int64_t n = static_cast<int64_t>(blockIdx.x) * kDecodeWarps + (threadIdx.x >> 5);
  if (n >= N) return;  // whole warp
  const int col = blockIdx.y * (32 * VEC) + lane * VEC;
  const bool active = col < D;
  const int colc = active ? col : 0;
  int myid = lane < LC ? __ldg(ids + n * LC + lane) : 0;
  bool bad = false;
  while (true) {
    Gather<CB_BF16, VEC> g[LC];
    bool use[LC];
#pragma unroll
    for (int l = 0; l < LC; ++l) {
      const int id = __shfl_sync(0xffffffffu, myid, l);
      const bool ok = static_cast<unsigned>(id) < static_cast<unsigned>(K);
      bad |= !ok;
      use[l] = ok;
      g[l].load(cb, (static_cast<int64_t>(l) * K + (ok ? id : 0)) * D + colc);
    }
    const int64_t nn = n + stride;
    const int nextid = (lane < LC && nn < N) ? __ldg(ids + nn * LC + lane) : 0;
    float acc[VEC];
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
#pragma unroll
    for (int l = 0; l < LC; ++l)
      if (use[l]) g[l].add_to(acc);
    if (active) {
      float4 *dst = reinterpret_cast<float4 *>(recon + n * D + col);
#pragma unroll
      for (int k = 0; k < VEC; k += 4) __stcs(dst + k / 4, make_float4(acc[k], acc[k + 1], acc[k + 2], acc[k + 3]));
    }
    if (nn >= N) break;
    n = nn;
    myid = nextid;
  }
  if (bad && lane == 0 && blockIdx.y == 0) set_status(status, RVQ_ERR_ID_RANGE);
}

// ---------------------------------------------------------------- TMA gather decode (bf16)
//
// Optional path (RVQ_DECODE_TMA=1) for bf16 codebooks with D % 256 == 0 and L <= 16: the codeword
// rows of a token are fetched by
// the tensor memory accelerator (cp.async.bulk.tensor tile::gather4: four rows of one 256-column
// slice per instruction) into a per-warp shared-memory ring, so every warp keeps kTmaDepth tokens'
// rows in flight without holding them in registers.  Each warp is its own pipeline: lane 0 issues,
// all 32 lanes wait on the stage's mbarrier, sum the rows (8 columns per lane, ascending level
// order, fp32) and stream the result to recon.  An id outside [0, K) fetches row 0 of its level
// and is left out of the sum.
constexpr int kTmaWarps = 8;
constexpr int kTmaCols = 256;           // columns per slice = the gather box width
constexpr int kTmaRing = 24576;         // ring bytes per warp

template <int LC>
struct TmaCfg {
  static constexpr int G4 = (LC + 3) / 4;                // gather4 loads per token
  static constexpr int STAGE = G4 * 4 * kTmaCols * 2;    // bytes per token (padding rows fetch row 0)
  static constexpr int DEPTH = kTmaRing / STAGE >= 2 ? kTmaRing / STAGE : 2;
  static constexpr int WARP_BYTES = DEPTH * STAGE;
  static constexpr int SMEM = kTmaWarps * WARP_BYTES + 1024;  // + alignment slack
  static_assert(SMEM <= 232448, "decode ring above the per-block shared-memory limit");
};

__device__ __forceinline__ void tma_gather4(const CUtensorMap *m, uint64_t *bar, void *dst, int32_t x, int32_t r0,
                                            int32_t r1, int32_t r2, int32_t r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}

template <int LC>
__global__ void __launch_bounds__(kTmaWarps * 32, 1)
    decode_tma_kernel(const __grid_constant__ CUtensorMap tm, const int32_t *__restrict__ ids, int64_t N, int K,
                      int D, float *__restrict__ recon, int32_t *status) {
  using C = TmaCfg<LC>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kTmaWarps][C::DEPTH];
  __shared__ int abort_flag;
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0)
    for (int s = 0; s < C::DEPTH; ++s) mbar_init(&full[warp][s], 1);
  fence_mbar_init();
  __syncthreads();
  griddep_launch_dependents();
  griddep_wait();
  if (threadIdx.x == 0) tma_prefetch_desc(&tm);
  uint8_t *ring = smem + warp * C::WARP_BYTES;
  const int x = blockIdx.y * kTmaCols;
  const int col = x + lane * 8;
  const bool active = col < D;
  // this warp's tokens: n = gw + t * GW for t = 0 .. cnt-1
  const int64_t GW = static_cast<int64_t>(gridDim.x) * kTmaWarps;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kTmaWarps + warp;
  const int64_t cnt = gw < N ? (N - 1 - gw) / GW + 1 : 0;
  // ids of tokens [32b, 32b + 32): lane j holds token 32b + j's ids (idA: current block, idB: next)
  int idA[LC], idB[LC];
  auto load_block = [&](int64_t b, int (&dst)[LC]) {
    const int64_t t = b * 32 + lane;
    const int64_t n = gw + t * GW;
#pragma unroll
    for (int l = 0; l < LC; ++l) dst[l] = t < cnt ? __ldg(ids + n * LC + l) : 0;
  };
  load_block(0, idA);
  load_block(1, idB);
  bool bad = false;
  // token t's ids, from the lane that holds them (block cur_block in idA, the next one in idB)
  auto fetch_ids = [&](int64_t t, int64_t cur_block, int (&out)[LC]) {
    const int src = static_cast<int>(t & 31);
    const bool next = (t >> 5) != cur_block;
#pragma unroll
    for (int l = 0; l < LC; ++l) {
      const int a = __shfl_sync(0xffffffffu, idA[l], src);
      const int b = __shfl_sync(0xffffffffu, idB[l], src);
      out[l] = next ? b : a;
    }
  };
  // lane 0 issues token t into stage t % DEPTH
  auto issue_token = [&](int64_t t, const int (&tid)[LC]) {
    const int s = static_cast<int>(t % C::DEPTH);
    uint8_t *dst = ring + s * C::STAGE;
    int32_t row[C::G4 * 4];
#pragma unroll
    for (int l = 0; l < C::G4 * 4; ++l) {
      const bool real = l < LC;
      const int id = real ? tid[l] : 0;
      const bool ok = static_cast<unsigned>(id) < static_cast<unsigned>(K);
      bad |= real && !ok;
      row[l] = (real ? l : 0) * K + (ok ? id : 0);
    }
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&full[warp][s], C::STAGE);
#pragma unroll
    for (int q = 0; q < C::G4; ++q)
      tma_gather4(&tm, &full[warp][s], dst + q * 4 * kTmaCols * 2, x, row[4 * q], row[4 * q + 1], row[4 * q + 2],
                  row[4 * q + 3]);
  };
  // prologue: the first DEPTH tokens (all in block 0: DEPTH < 32)
  static_assert(C::DEPTH < 32, "the prologue takes its ids from the first block of 32 tokens");
  int64_t issued = 0;
  for (int64_t t = 0; t < C::DEPTH && t < cnt; ++t) {
    int tid[LC];
    fetch_ids(t, 0, tid);
    if (lane == 0) issue_token(t, tid);
    ++issued;
  }
  bool ok = true;
  for (int64_t t = 0; t < cnt; ++t) {
    const int64_t blk = t >> 5;
    const int s = static_cast<int>(t % C::DEPTH);
    const uint32_t parity = static_cast<uint32_t>((t / C::DEPTH) & 1);
    int tid[LC];
    fetch_ids(t, blk, tid);  // this token's ids (validity of each row)
    if (!mbar_wait(&full[warp][s], parity, &abort_flag)) {
      ok = false;
      break;
    }
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    const uint8_t *st = ring + s * C::STAGE + lane * 16;
#pragma unroll
    for (int l = 0; l < LC; ++l) {
      const uint4 raw = *reinterpret_cast<const uint4 *>(st + l * kTmaCols * 2);
      if (static_cast<unsigned>(tid[l]) < static_cast<unsigned>(K)) {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
          acc[2 * k] += f.x;
          acc[2 * k + 1] += f.y;
        }
      }
    }
    if (active) {
      float4 *dst = reinterpret_cast<float4 *>(recon + (gw + t * GW) * D + col);
      __stcs(dst, make_float4(acc[0], acc[1], acc[2], acc[3]));
      __stcs(dst + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
    }
    fence_proxy_async_smem();  // this lane's reads of stage s are ordered before its refill
    __syncwarp();
    const int64_t tn = t + C::DEPTH;
    if (tn < cnt) {
      int nid[LC];
      fetch_ids(tn, blk, nid);
      if (lane == 0) issue_token(tn, nid);
      ++issued;
    }
    if ((t & 31) == 31) {  // the next block becomes current; load the one after it
#pragma unroll
      for (int l = 0; l < LC; ++l) idA[l] = idB[l];
      load_block(blk + 2, idB);
    }
  }
  if (!ok) {
    abort_flag = 1;
    set_status(status, RVQ_ERR_TIMEOUT);
    // no bulk copy may still be in flight when the block exits: wait (bounded) for the issued ones
    if (lane == 0) {
      int never = 0;
      for (int64_t t = issued - C::DEPTH < 0 ? 0 : issued - C::DEPTH; t < issued; ++t)
        mbar_wait(&full[warp][static_cast<int>(t % C::DEPTH)], static_cast<uint32_t>((t / C::DEPTH) & 1), &never);
    }
  }
  if (bad && blockIdx.y == 0) set_status(status, RVQ_ERR_ID_RANGE);
}

typedef CUresult (*DecodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline DecodeTiledFn decode_tiled_fn() {
  static DecodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<DecodeTiledFn>(p);
  });
  return fn;
}

// RVQ_DECODE_TMA=1 selects the TMA gather kernel for bf16 codebooks (tuning knob; off by default:
// on 2^20 tokens x 8 levels of [8,16384,1024] bf16 codebooks it took 3.13 ms against 1.76 ms for
// the register-gather kernel).
inline bool tma_decode_enabled() {
  static int v = [] {
    const char *e = getenv("RVQ_DECODE_TMA");
    return e ? atoi(e) : 0;
  }();
  return v != 0;
}

template <int LC>
cudaError_t launch_tma_t(const int32_t *ids, int64_t N, const void *cb, int K, int D, float *recon, int32_t *status,
                         cudaStream_t s) {
  using C = TmaCfg<LC>;
  DecodeTiledFn fn = decode_tiled_fn();
  if (!fn) return cudaErrorUnknown;
  static int attr_ok = -1;
  if (attr_ok < 0)
    attr_ok = cudaFuncSetAttribute(decode_tma_kernel<LC>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) ==
              cudaSuccess;
  if (attr_ok != 1) return cudaErrorUnknown;
  CUtensorMap tm;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(LC) * K};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {kTmaCols, 1};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(cb), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorUnknown;
  int sms = 0;
  if (device_sm_count(&sms) != RVQ_OK) return cudaErrorUnknown;
  const int64_t gx = std::min<int64_t>((N + kTmaWarps - 1) / kTmaWarps, sms);
  const int gy = D / kTmaCols;
  if (gy > 65535) return cudaErrorInvalidValue;
  return launch_pdl(decode_tma_kernel<LC>, dim3(static_cast<unsigned>(gx), gy), dim3(kTmaWarps * 32),
                    static_cast<size_t>(C::SMEM), s, tm, ids, N, K, D, recon, status);
}

template <int LC = 1>
cudaError_t dispatch_tma(int L, const int32_t *ids, int64_t N, const void *cb, int K, int D, float *recon,
                         int32_t *status, cudaStream_t s) {
  if constexpr (LC > 16) {
    return cudaErrorInvalidValue;
  } else {
    if (L == LC) return launch_tma_t<LC>(ids, N, cb, K, D, recon, status, s);
    return dispatch_tma<LC + 1>(L, ids, N, cb, K, D, recon, status, s);
  }
}

template <bool CB_BF16, int VEC, int LC>
cudaError_t launch_fixed(const int32_t *ids, int64_t N, const void *cb, int K, int D, float *recon, int32_t *status,
                         cudaStream_t s) {
  // per slice, enough blocks to fill every SM at the kernel's occupancy (6 blocks of 8 warps);
  // each warp then walks rows with a stride of the slice's warp count
  int sms = 0;
  if (device_sm_count(&sms) != RVQ_OK) return cudaErrorUnknown;
  const int64_t gx = std::min<int64_t>((N + kDecodeWarps - 1) / kDecodeWarps, static_cast<int64_t>(sms) * kDecodeBlocksPerSm);
  const int gy = (D + 32 * VEC - 1) / (32 * VEC);
  if (gx > 0x7FFFFFFFLL || gy > 65535) return cudaErrorInvalidValue;
  return launch_pdl(decode_fixed_kernel<CB_BF16, VEC, LC>, dim3(static_cast<unsigned>(gx), gy),
                    dim3(kDecodeWarps * 32), 0, s, ids, N, cb, K, D, recon, status);
}

template <bool CB_BF16, int VEC, int LC = 1>
cudaError_t dispatch_fixed(int L, const int32_t *ids, int64_t N, const void *cb, int K, int D, float *recon,
                           int32_t *status, cudaStream_t s) {
  if constexpr (LC > 16) {
    return cudaErrorInvalidValue;
  } else {
    if (L == LC) return launch_fixed<CB_BF16, VEC, LC>(ids, N, cb, K, D, recon, status, s);
    return dispatch_fixed<CB_BF16, VEC, LC + 1>(L, ids, N, cb, K, D, recon, status, s);
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
    // the TMA gather needs whole 256-column slices, a row coordinate range within int32, and rows
    // addressable as a 2-D tensor (16-byte aligned base, checked by the caller)
    if (cb_dtype == RVQ_BF16 && D % kTmaCols == 0 && static_cast<int64_t>(L) * K < (int64_t(1) << 31) &&
        tma_decode_enabled()) {
      e = dispatch_tma(L, ids, N, cb, K, D, recon, status, s);
      note_launch();
      return e == cudaSuccess ? RVQ_OK : e == cudaErrorInvalidValue ? RVQ_ERR_UNSUPPORTED : RVQ_ERR_CUDA;
    }
    if (cb_dtype == RVQ_BF16)
      e = (D % 8 == 0 && kBf16Vec == 8) ? dispatch_fixed<true, 8>(L, ids, N, cb, K, D, recon, status, s)
                                        : dispatch_fixed<true, 4>(L, ids, N, cb, K, D, recon, status, s);
    else
      e = dispatch_fixed<false, 4>(L, ids, N, cb, K, D, recon, status, s);
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
