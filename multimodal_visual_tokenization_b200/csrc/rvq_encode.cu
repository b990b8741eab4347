// rvq_encode.cu -- greedy residual vector quantization on sm_100a.
//
// Method (LongCat-2.5 technical blog, "Visual Primitive Modeling" -> "Discrete Native
// Resolution Vision Transformer": RVQ over native-resolution encoder features; Meituan
// LongCat-2.5 open-source article, "02 Visual Coding and 3D": detail is added level by
// level): for every level l, every row takes the codeword nearest (squared Euclidean, lowest
// index on ties) to its running residual and subtracts it.
//
// Engine.  Both paths score with the same distance GEMM tile: s = r~ . c~ for a 128-row x 256-codeword
// tile as a dense bf16 GEMM with fp32 accumulation, operands moved by TMA (cp.async.bulk.tensor,
// 128B swizzle) into a shared-memory ring, tcgen05.mma issued by one thread into a double-buffered
// TMEM accumulator (2 x 256 columns).  One extra K=16 step adds ||c||^2/2 (split into three bf16
// parts) and the main steps negate A, so TMEM holds d~/2 = ||c||^2/2 - r~.c~ directly.  Epilogue
// warps read it with tcgen05.ld (one TMEM lane = one row) and keep a running top-8 (d~, id) per
// row; the distance matrix never leaves the SM.
//
//  * encode_flow_kernel (D in (128, 256] or (512, 1024]): every level in ONE launch with every
//    CTA resident (cooperative for single CTAs), one CTA per SM.  The level loop is a dataflow
//    over 128-row tiles: GEMM chunks of (level l, row tile rt) start as soon as the certificate
//    warps have settled level l-1 of rt (counter cert_done[l-1][rt]); the certificate warps take
//    (l, rt) once all its chunks are written (chunk_done[l][rt]).  Per CTA: a TMA producer warp,
//    an MMA-issuer warp, a norm-split warp, 4 epilogue + 4 certificate warps (D in (512, 1024]) or
//    8 + 3 (D in (128, 256]).  For D in (512, 1024] and batches of at least kPairMinRows rows the
//    CTAs run as pairs (2-CTA clusters, tcgen05 cta_group::2): each CTA loads its own 128 rows and
//    half of every 256-codeword tile, the leader issues M = 256 MMAs, and each CTA's TMEM holds its
//    own rows' accumulators, so an SM streams 32 KB instead of 48 KB per K step.  Rows the certificate cannot settle get an
//    exact scan of all K codewords, cut into slices any certificate warp may run.  Every wait is
//    bounded (status RVQ_ERR_TIMEOUT when nothing moved for two seconds).
//  * other widths (and RVQ_PERSISTENT=0): per level, dist_topk_kernel (persistent GEMM + top-8 over
//    contiguous ranges of (row tile, codeword tile) units, 4 or 8 epilogue warps), then
//    rescore_fast_kernel / rescore_kernel (certificate, one warp per row) and
//    fallback_fast_kernel / fallback_kernel (exact scan of the rows the certificate left).
//
// Certificate (rescore_row): the candidate lists of a row are merged, every approximate distance
// carries the bf16 error bound E below, every candidate within 2E of the best is rescored exactly
// (fp32 differences, fp64 sums), and the exact minimum (ties: lowest id) is accepted when
// best - ||r||^2 < T - E, T being the smallest approximate distance some list dropped.  Accepted
// rows update r -= C_l[id] in fp32 and write the next level's bf16 operand and row statistics.
//
// Error bound, per row and level (r fp32 residual, r~ = bf16(r), c stored codeword, c~ = bf16(c),
// n = fl32(||c||^2), gamma = (D+32) 2^-22; Cmax, dCmax, C~max, Nmax the per-level maxima of ||c||,
// ||c-c~||, ||c~||, n from rvq_build_norms):
//   | (||r-c||^2 - ||r||^2) - d~ | <= (D/32+2) 2^-24 Nmax + 2 (||r-r~|| Cmax + ||r~|| dCmax)
//                                     + 2 gamma (||r~|| C~max + 0.51 Nmax) + 2^-23 Nmax
// (Cauchy-Schwarz on the two rounding-error vectors, a worst-case bound of fp32 accumulation of
// D products and three norm parts with truncation allowed, the fp32 norm sums and the three-part
// bf16 split of n/2), inflated by 1%.  It assumes that the tensor core forms bf16 products
// exactly and adds them into the fp32 accumulator with at most one rounding (or truncation) per
// addition; a GPU test measures |d~ - exact| against E on the workloads.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {

int launch_decode(const int32_t *ids, int64_t N, int L, const void *cb, int cb_dtype, int K, int D, float *recon,
                  int32_t *status, cudaStream_t s);

namespace enc {

constexpr int BM = 128;       // rows per tile (TMEM lanes)
constexpr int BN = 256;       // codewords per tile (UMMA N)
constexpr int BK = 64;        // bf16 elements per k-block = one 128-byte swizzle row
constexpr int UK = 16;        // K of one kind::f16 UMMA
constexpr int TOPK = 8;
constexpr int MAX_SLOTS = 16;  // partial lists per row tile (bounds the rescore merge)
constexpr int CPL = MAX_SLOTS * TOPK / 32;  // candidates per lane when one warp merges a row's lists
constexpr int A_BYTES = BM * BK * 2;
constexpr int TMEM_COLS = 2 * BN;
// Norm term of the distance, folded into the GEMM as one extra K=16 step: A_aug rows are
// (1, 1, 1, 0, ..., 0) and B_aug row j holds ||c_j||^2 / 2 split into three bf16 parts, so the
// accumulator gets ||c_j||^2 / 2 on top of -r~.c~_j (the main steps negate A).  Both aug tiles
// are K-major without swizzle: 8-row x 16-byte core matrices.
constexpr int AUG_A_BYTES = (BM / 8) * 256;       // row groups 256 B apart, K halves 128 B apart
constexpr int AUG_B_BYTES = (BN / 8) * 128 + 128;  // K half 1 aliases the next group (A's half 1 is 0)
constexpr uint16_t BF16_ONE = 0x3F80;
constexpr uint16_t BF16_BIG = 0x7F7F;  // largest finite bf16: codeword columns past K

__device__ __forceinline__ float inf_f() { return __int_as_float(0x7f800000); }
constexpr float kPastK = 3.0e38f;  // key of a column past K (never a real half-distance)
constexpr int kMergeLanes = 10;  // lanes needing inserts that switch a chunk to merging
__device__ __forceinline__ double inf_d() { return __longlong_as_double(0x7ff0000000000000LL); }

// Thread organisation of the distance-GEMM block: EPI epilogue warps (EPI/4 column groups x 4
// TMEM lane quadrants), then the TMA producer warp, the MMA-issuer warp and the norm-split warp.
template <int EPI>
struct GemmCfg {
  static constexpr int GROUPS = EPI / 4;
  static constexpr int COLS = BN / GROUPS;  // columns of a tile one epilogue thread scans
  static constexpr int CHUNKS = COLS / 32;
  static constexpr int EPI_THREADS = EPI * 32;
  static constexpr int THREADS = EPI_THREADS + 96;
  static constexpr int PRODUCER = EPI;
  static constexpr int ISSUER = EPI + 1;
  static constexpr int SPLITTER = EPI + 2;
  static constexpr int STAGE = A_BYTES + BN * BK * 2;
  static constexpr int NSTAGE = EPI >= 16 ? 3 : 4;
  static constexpr int AUG_A_OFF = NSTAGE * STAGE;
  static constexpr int AUG_B_OFF = AUG_A_OFF + AUG_A_BYTES;                // 2 slots
  static constexpr int MERGE_OFF = AUG_B_OFF + 2 * AUG_B_BYTES;            // (GROUPS-1) x 128 x 8 x 8 B
  static constexpr int BAR_OFF = MERGE_OFF + (GROUPS - 1) * BM * TOPK * 8;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;                        // + barriers + alignment slack
  static_assert(SMEM <= 232448, "dynamic shared memory above the 227 KB per-block limit");
};

struct GemmArgs {
  const float *norms;  // [K] of this level
  int64_t N;
  int K;
  int D;
  int64_t U;  // units = row tiles x codeword tiles
  int Tc;     // codeword tiles
  int G;      // CTAs
  int maxs;   // partial-list slots per row tile
  float2 *cand;
  int32_t *status;
  int32_t *zero_counter;  // set to 0 by the first thread (the level's fallback counter), or null
};
// Units are (row tile, codeword tile) pairs of 128 rows x 256 codewords; the U units are split into
// G contiguous ranges, one per CTA.

// CTA that owns unit u when U units are split into G contiguous ranges [cU/G, (c+1)U/G).
__host__ __device__ __forceinline__ int cta_of_unit(int64_t u, int64_t U, int G) {
  return static_cast<int>(((u + 1) * static_cast<int64_t>(G) - 1) / U);
}

// Insert (x, ix) into the ascending list bd/bi, dropping the largest entry.  Entries equal to x
// stay ahead of it (first seen wins).  Written as independent compares + selects so the update
// has a short dependency chain.
__device__ __forceinline__ void topk_insert(float (&bd)[TOPK], int (&bi)[TOPK], float x, int ix) {
  bool c[TOPK];
#pragma unroll
  for (int t = 0; t < TOPK; ++t) c[t] = bd[t] <= x;
#pragma unroll
  for (int t = TOPK - 1; t >= 1; --t) {
    const float nb = c[t] ? bd[t] : (c[t - 1] ? x : bd[t - 1]);
    const int ni = c[t] ? bi[t] : (c[t - 1] ? ix : bi[t - 1]);
    bd[t] = nb;
    bi[t] = ni;
  }
  if (!c[0]) {
    bd[0] = x;
    bi[0] = ix;
  }
}

// ---- branch-free top-8 of a 32-value chunk, used when many lanes of a warp need inserts at once.
// Keys carry the chunk-local index in their 5 low mantissa bits (a relative perturbation below
// 2^-18, covered by the certificate's error bound), so compare-exchanges are two min/max ops.
__device__ __forceinline__ void cx(float &a, float &b) {
  const float lo = fminf(a, b);
  b = fmaxf(a, b);
  a = lo;
}
// Batcher odd-even merge sort of 8 keys, ascending (19 compare-exchanges).
__device__ __forceinline__ void sort8(float *v) {
  cx(v[0], v[1]); cx(v[2], v[3]); cx(v[4], v[5]); cx(v[6], v[7]);
  cx(v[0], v[2]); cx(v[1], v[3]); cx(v[4], v[6]); cx(v[5], v[7]);
  cx(v[1], v[2]); cx(v[5], v[6]);
  cx(v[0], v[4]); cx(v[1], v[5]); cx(v[2], v[6]); cx(v[3], v[7]);
  cx(v[2], v[4]); cx(v[3], v[5]);
  cx(v[1], v[2]); cx(v[3], v[4]); cx(v[5], v[6]);
}
// Smallest 8 of two ascending 8-lists, ascending: elementwise min against the reversed second
// list gives a bitonic sequence, which three half-cleaner stages sort.
__device__ __forceinline__ void merge8(float *a, const float *b) {
#pragma unroll
  for (int t = 0; t < 8; ++t) a[t] = fminf(a[t], b[7 - t]);
  cx(a[0], a[4]); cx(a[1], a[5]); cx(a[2], a[6]); cx(a[3], a[7]);
  cx(a[0], a[2]); cx(a[1], a[3]); cx(a[4], a[6]); cx(a[5], a[7]);
  cx(a[0], a[1]); cx(a[2], a[3]); cx(a[4], a[5]); cx(a[6], a[7]);
}
__device__ __forceinline__ void cx_idx(float &a, float &b, int &ia, int &ib) {
  const bool sw = b < a;
  const float ta = a;
  const int tia = ia;
  a = sw ? b : a;
  b = sw ? ta : b;
  ia = sw ? ib : ia;
  ib = sw ? tia : ib;
}
// Merge the chunk of 32 keys d[] (columns c0 + j, all finite) into the running list.
// d[j] for a run-time j in [0, 32) as a tree of selects (no local-memory copy of d).
__device__ __forceinline__ float pick32(const float (&d)[32], int j) {
  float t16[16], t8[8], t4[4], t2[2];
#pragma unroll
  for (int i = 0; i < 16; ++i) t16[i] = (j & 1) ? d[2 * i + 1] : d[2 * i];
#pragma unroll
  for (int i = 0; i < 8; ++i) t8[i] = (j & 2) ? t16[2 * i + 1] : t16[2 * i];
#pragma unroll
  for (int i = 0; i < 4; ++i) t4[i] = (j & 4) ? t8[2 * i + 1] : t8[2 * i];
#pragma unroll
  for (int i = 0; i < 2; ++i) t2[i] = (j & 8) ? t4[2 * i + 1] : t4[2 * i];
  return (j & 16) ? t2[1] : t2[0];
}

// Insert the chunk entries below the current 8th best, in column order (the same result as
// offering all 32 to topk_insert in order).  The entries are found from a bit mask and fetched
// with pick32, so the loop runs as often as the busiest lane has entries and stays small in code.
__device__ __forceinline__ void topk_insert_few(float (&bd)[TOPK], int (&bi)[TOPK], const float (&d)[32], int c0) {
  const float thr = bd[TOPK - 1];
  unsigned mask = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) mask |= (d[j] < thr ? 1u : 0u) << j;
#pragma unroll 1
  while (__any_sync(0xffffffffu, mask != 0)) {
    const int j = __ffs(mask) - 1;
    mask &= mask - 1;
    if (j >= 0) topk_insert(bd, bi, pick32(d, j), c0 + j);
  }
}

__device__ __forceinline__ void topk_merge_chunk(float (&bd)[TOPK], int (&bi)[TOPK], const float (&d)[32], int c0) {
  float k[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) k[j] = __uint_as_float((__float_as_uint(d[j]) & ~31u) | static_cast<uint32_t>(j));
  sort8(k);
  sort8(k + 8);
  sort8(k + 16);
  sort8(k + 24);
  merge8(k, k + 8);
  merge8(k + 16, k + 24);
  merge8(k, k + 16);  // k[0..7]: the chunk's 8 smallest keys, ascending
  float cv[TOPK];
  int ci[TOPK];
#pragma unroll
  for (int t = 0; t < TOPK; ++t) {
    const float q = k[TOPK - 1 - t];
    const int qi = c0 + static_cast<int>(__float_as_uint(q) & 31u);
    const bool keep = bd[t] <= q;
    cv[t] = keep ? bd[t] : q;
    ci[t] = keep ? bi[t] : qi;
  }
  cx_idx(cv[0], cv[4], ci[0], ci[4]); cx_idx(cv[1], cv[5], ci[1], ci[5]);
  cx_idx(cv[2], cv[6], ci[2], ci[6]); cx_idx(cv[3], cv[7], ci[3], ci[7]);
  cx_idx(cv[0], cv[2], ci[0], ci[2]); cx_idx(cv[1], cv[3], ci[1], ci[3]);
  cx_idx(cv[4], cv[6], ci[4], ci[6]); cx_idx(cv[5], cv[7], ci[5], ci[7]);
  cx_idx(cv[0], cv[1], ci[0], ci[1]); cx_idx(cv[2], cv[3], ci[2], ci[3]);
  cx_idx(cv[4], cv[5], ci[4], ci[5]); cx_idx(cv[6], cv[7], ci[6], ci[7]);
#pragma unroll
  for (int t = 0; t < TOPK; ++t) {
    bd[t] = cv[t];
    bi[t] = ci[t];
  }
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t *>(&b);
}
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

template <int EPI>
__global__ void __launch_bounds__(GemmCfg<EPI>::THREADS, 1)
    dist_topk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmArgs a) {
  using C = GemmCfg<EPI>;
  constexpr int NSTAGE = C::NSTAGE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *aug_a = smem + C::AUG_A_OFF;
  uint8_t *aug_b = smem + C::AUG_B_OFF;
  float2 *mbuf = reinterpret_cast<float2 *>(smem + C::MERGE_OFF);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *empty = full + NSTAGE;
  uint64_t *tfull = empty + NSTAGE;
  uint64_t *tempty = tfull + 2;
  uint64_t *afull = tempty + 2;
  uint64_t *mready = afull + 2;
  uint64_t *mdone = mready + 1;
  uint64_t *mma_done = mdone + 1;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  volatile int *never = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t cid = blockIdx.x;
  const int64_t u0 = cid * a.U / a.G;
  const int64_t u1 = (cid + 1) * a.U / a.G;
  const int KB = a.D / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::EPI_THREADS);
      mbar_init(&afull[b], 32);
    }
    mbar_init(mready, C::EPI_THREADS - 128 > 0 ? C::EPI_THREADS - 128 : 1);
    mbar_init(mdone, 128);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbar_init();
  }
  // constant aug tiles: A_aug rows (1,1,1,0,...) and zeros everywhere else
  for (int i = threadIdx.x; i < (AUG_A_BYTES + 2 * AUG_B_BYTES) / 16; i += blockDim.x) {
    uint4 v = make_uint4(0, 0, 0, 0);
    if (i < AUG_A_BYTES / 16 && ((i * 16) % 256) < 128)  // K half 0 of a row: elements 0..2 are one
      v = make_uint4(BF16_ONE | (static_cast<uint32_t>(BF16_ONE) << 16), BF16_ONE, 0, 0);
    reinterpret_cast<uint4 *>(aug_a)[i] = v;
  }
  fence_proxy_async_smem();
  if (warp == C::ISSUER) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  griddep_launch_dependents();
  griddep_wait();  // the residual operand and candidate buffers belong to the previous kernel until here
  if (a.zero_counter && blockIdx.x == 0 && threadIdx.x == 0) *a.zero_counter = 0;

  if (warp == C::PRODUCER) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int64_t u = u0; u < u1 && ok; ++u) {
        const int64_t rt = u / a.Tc;
        const int ct = static_cast<int>(u - rt * a.Tc);
        const int32_t row0 = static_cast<int32_t>(rt * BM);
        const int32_t cw0 = ct * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *sa = smem + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], C::STAGE);
          tma_load_2d(&tmA, &full[s], sa, kb * BK, row0);
          tma_load_2d(&tmB, &full[s], sa + A_BYTES, kb * BK, cw0);
          ++issued;
          if (++s == NSTAGE) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(a.status, RVQ_ERR_TIMEOUT);
        // no bulk copy may still be landing in shared memory when the block exits
        const int64_t pending = issued < NSTAGE ? issued : NSTAGE;
        for (int64_t j = 0; j < pending; ++j) {
          int back = s - 1 - static_cast<int>(j);
          uint32_t p = ph;
          while (back < 0) {
            back += NSTAGE;
            p ^= 1u;
          }
          mbar_wait(&full[back], p, never);
        }
      }
    }
  } else if (warp == C::SPLITTER) {
    // ------------------------------------------------------------ norm split -> B_aug tiles
    int64_t i = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1; ++u, ++i) {
      const int slot = static_cast<int>(i & 1);
      const int ct = static_cast<int>(u - (u / a.Tc) * a.Tc);
      constexpr int GROUPS_B = BN / 8;  // row groups of the tile
      const bool writer = lane < GROUPS_B;
      const int c0 = ct * BN + lane * 8;  // row group `lane`
      float h[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) h[j] = (writer && c0 + j < a.K) ? 0.5f * __ldg(a.norms + c0 + j) : 0.f;
      // the slot is free once the MMAs of the unit two back (same slot) have completed
      bool got = i < 2 || mbar_wait(&tfull[slot], static_cast<uint32_t>(((i >> 1) - 1) & 1), abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      uint4 *dst = reinterpret_cast<uint4 *>(aug_b + slot * AUG_B_BYTES + lane * 128);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!writer) break;
        uint16_t h1, h2 = 0, h3 = 0;
        if (c0 + j < a.K) {
          h1 = bf16_bits_rn(h[j]);
          const float r1 = h[j] - bf16_bits_to_float(h1);  // exact
          h2 = bf16_bits_rn(r1);
          const float r2 = r1 - bf16_bits_to_float(h2);    // exact
          h3 = bf16_bits_rn(r2);
        } else {
          h1 = BF16_BIG;
        }
        dst[j] = make_uint4(h1 | (static_cast<uint32_t>(h2) << 16), h3, 0, 0);
      }
      fence_proxy_async_smem();
      mbar_arrive(&afull[slot]);
    }
    if (!ok) {
      *abort_flag = 1;
      set_status(a.status, RVQ_ERR_TIMEOUT);
    }
  } else if (warp == C::ISSUER) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_main = idesc_bf16_f32(BM, BN, true);  // accumulates -r~.c~
      constexpr uint32_t idesc_aug = idesc_bf16_f32(BM, BN, false);  // + ||c||^2 / 2
      const uint64_t adesc_aug = sdesc_k_noswizzle(smem_u32(aug_a), 128, 256);
      int s = 0;
      uint32_t ph = 0;
      int64_t i = 0;
      bool ok = true;
      for (int64_t u = u0; u < u1 && ok; ++u, ++i) {
        const int buf = static_cast<int>(i & 1);
        const uint32_t tph = static_cast<uint32_t>((i >> 1) & 1);
        if (!mbar_wait(&tempty[buf], tph ^ 1u, abort_flag) || !mbar_wait(&afull[buf], tph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem_base + static_cast<uint32_t>(buf * BN);
        const uint64_t bdesc_aug = sdesc_k_noswizzle(smem_u32(aug_b + buf * AUG_B_BYTES), 128, 128);
        umma_f16(dt, adesc_aug, bdesc_aug, idesc_aug, 0u);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE);
          const uint64_t ad = sdesc_k128(sa);
          const uint64_t bd = sdesc_k128(sa + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UK; ++k) {
            const uint64_t step = static_cast<uint64_t>(k * UK * 2 / 16);
            umma_f16(dt, ad + step, bd + step, idesc_main, 1u);
          }
          umma_commit(&empty[s]);
          if (++s == NSTAGE) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[buf]);
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(a.status, RVQ_ERR_TIMEOUT);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, never);
    }
  } else {
    // ------------------------------------------------------------ epilogue: running top-8
    // TMEM holds half the shifted distance, ||c||^2/2 - r~.c~ = d~/2; lists keep d~/2 and are
    // doubled (exactly) when written out.
    const int quad = warp & 3;
    const int grp = warp >> 2;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    float bd[TOPK];
    int bi[TOPK];
#pragma unroll
    for (int t = 0; t < TOPK; ++t) {
      bd[t] = inf_f();
      bi[t] = -1;
    }
    int64_t cur_rt = -1;
    int64_t i = 0;
    uint32_t nflush = 0;
    bool ok = true;

    // Merge the column groups' lists of row tile rt (group 0 gathers) and write it to this CTA's slot.
    auto flush = [&](int64_t rt) -> bool {
      if constexpr (C::GROUPS > 1) {
        float2 *mine = mbuf + (static_cast<int64_t>(grp - 1) * BM + row_in_tile) * TOPK;
        if (grp > 0) {
          if (nflush > 0 && !mbar_wait(mdone, (nflush - 1) & 1u, abort_flag)) return false;
#pragma unroll
          for (int t = 0; t < TOPK; ++t) mine[t] = make_float2(bd[t], __int_as_float(bi[t]));
          mbar_arrive(mready);
        } else {
          if (!mbar_wait(mready, nflush & 1u, abort_flag)) return false;
          #pragma unroll 1
          for (int e8 = 0; e8 < (C::GROUPS - 1) * TOPK; ++e8) {
            const float2 e = mbuf[(static_cast<int64_t>(e8 / TOPK) * BM + row_in_tile) * TOPK + e8 % TOPK];
            if (e.x < bd[TOPK - 1]) topk_insert(bd, bi, e.x, __float_as_int(e.y));
          }
          mbar_arrive(mdone);
        }
      }
      ++nflush;
      if (grp == 0) {
        const int64_t n = rt * BM + row_in_tile;
        if (n < a.N) {
          const int slot = static_cast<int>(cid) - cta_of_unit(rt * a.Tc, a.U, a.G);
          float4 *out = reinterpret_cast<float4 *>(a.cand + ((rt * a.maxs + slot) * BM + row_in_tile) * TOPK);
#pragma unroll
          for (int t = 0; t < TOPK; ++t)
            if (bi[t] >= a.K) {  // a past-K key kept only because the range had < 8 codewords
              bd[t] = inf_f();
              bi[t] = -1;
            }
#pragma unroll
          for (int t = 0; t < TOPK; t += 2)
            out[t / 2] =
                make_float4(2.f * bd[t], __int_as_float(bi[t]), 2.f * bd[t + 1], __int_as_float(bi[t + 1]));
        }
      }
      return true;
    };

    for (int64_t u = u0; u < u1; ++u, ++i) {
      const int64_t rt = u / a.Tc;
      const int ct = static_cast<int>(u - rt * a.Tc);
      if (rt != cur_rt) {
        if (cur_rt >= 0 && !flush(cur_rt)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int t = 0; t < TOPK; ++t) {
          bd[t] = inf_f();
          bi[t] = -1;
        }
        cur_rt = rt;
      }
      const int buf = static_cast<int>(i & 1);
      const uint32_t tph = static_cast<uint32_t>((i >> 1) & 1);
      const bool got = mbar_wait(&tfull[buf], tph, abort_flag);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int col0 = ct * BN;
      const int nvalid = min(BN, a.K - col0);
#pragma unroll 1
      for (int ch = 0; ch < C::CHUNKS; ++ch) {
        const int ct0 = grp * C::COLS + ch * 32;  // first column of the chunk within the tile
        uint32_t v[32];
        tmem_ld_32x32(lane_base + static_cast<uint32_t>(buf * BN + ct0), v);
        tmem_ld_wait();
        if (ch == C::CHUNKS - 1) {
          tc_fence_before();
          mbar_arrive(&tempty[buf]);
        }
        const int c0 = col0 + ct0;
        float d[32];
        if (ct0 + 32 <= nvalid) {
#pragma unroll
          for (int j = 0; j < 32; ++j) d[j] = __uint_as_float(v[j]);
        } else {  // columns past K: a large finite key (the merge path packs indices into keys)
#pragma unroll
          for (int j = 0; j < 32; ++j) d[j] = (ct0 + j < nvalid) ? __uint_as_float(v[j]) : kPastK;
        }
        // chunk minimum as a tree of 3-input minima (short dependency chain)
        float m11[11];
#pragma unroll
        for (int j = 0; j < 10; ++j) m11[j] = fmin3(d[3 * j], d[3 * j + 1], d[3 * j + 2]);
        m11[10] = fminf(d[30], d[31]);
        const float m4a = fmin3(m11[0], m11[1], m11[2]), m4b = fmin3(m11[3], m11[4], m11[5]);
        const float m4c = fmin3(m11[6], m11[7], m11[8]), m4d = fminf(m11[9], m11[10]);
        const float m = fminf(fmin3(m4a, m4b, m4c), m4d);
        const unsigned need = __ballot_sync(0xffffffffu, m < bd[TOPK - 1]);
        if (__popc(need) >= kMergeLanes) {
          topk_merge_chunk(bd, bi, d, c0);  // many lanes: one branch-free merge for the warp
        } else if (need) {
          topk_insert_few(bd, bi, d, c0);
        }
      }
    }
    if (ok && cur_rt >= 0 && !flush(cur_rt)) ok = false;
    if (!ok) {
      *abort_flag = 1;
      set_status(a.status, RVQ_ERR_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncwarp();
  __syncthreads();
  tc_fence_after();
  if (warp == C::ISSUER) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- row kernels

template <bool BF16>
__device__ __forceinline__ float4 ld4(const void *p, int64_t off) {
  if constexpr (BF16) {
    uint2 raw = __ldg(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p) + off));
    float2 x = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.x));
    float2 y = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.y));
    return make_float4(x.x, x.y, y.x, y.y);
  } else {
    return __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(p) + off));
  }
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_min_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ void store_bf16x4(__nv_bfloat16 *p, float4 v, float4 *rounded) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t *>(&a);
  packed.y = *reinterpret_cast<uint32_t *>(&b);
  *reinterpret_cast<uint2 *>(p) = packed;
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  *rounded = make_float4(fa.x, fa.y, fb.x, fb.y);
}

// r (fp32) -> bf16 operand row + (||r - r~||, ||r~||); one warp per row, lanes stride by 4.
__device__ __forceinline__ float2 write_operand_row(const float *r, __nv_bfloat16 *rt, int D, int lane) {
  float e2 = 0.f, q2 = 0.f;
  for (int i = lane * 4; i < D; i += 128) {
    const float4 v = *reinterpret_cast<const float4 *>(r + i);
    float4 q;
    store_bf16x4(rt + i, v, &q);
    const float ex = v.x - q.x, ey = v.y - q.y, ez = v.z - q.z, ew = v.w - q.w;
    e2 += ex * ex + ey * ey + ez * ez + ew * ew;
    q2 += q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
  }
  e2 = warp_sum_f(e2);
  q2 = warp_sum_f(q2);
  return make_float2(__fsqrt_ru(e2), __fsqrt_ru(q2));
}

// r_0 = fp32(x), its bf16 operand copy and row statistics; also clears the fallback counters
// and checks the packed-batch offsets.
template <bool X_BF16, bool WRITE_R>
__global__ void __launch_bounds__(256) init_kernel(const void *__restrict__ x, int64_t N, int D, float *__restrict__ R,
                                                   __nv_bfloat16 *__restrict__ Rt, float2 *__restrict__ rowstat,
                                                   int32_t *__restrict__ fb_count, int L,
                                                   const int64_t *__restrict__ offsets, int64_t B,
                                                   int32_t *status) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gtid < L) fb_count[gtid] = 0;
  if (offsets) {
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t b = gtid; b < B; b += nthreads)
      if (offsets[b] > offsets[b + 1]) set_status(status, RVQ_ERR_ARG);
    if (gtid == 0 && (offsets[0] != 0 || offsets[B] != N)) set_status(status, RVQ_ERR_ARG);
  }
  const int64_t n = gtid >> 5;
  if (n >= N) return;
  float e2 = 0.f, q2 = 0.f;
  for (int i = lane * 4; i < D; i += 128) {
    const float4 v = ld4<X_BF16>(x, n * D + i);
    if constexpr (WRITE_R) *reinterpret_cast<float4 *>(R + n * D + i) = v;
    float4 q;
    store_bf16x4(Rt + n * D + i, v, &q);
    const float ex = v.x - q.x, ey = v.y - q.y, ez = v.z - q.z, ew = v.w - q.w;
    e2 += ex * ex + ey * ey + ez * ez + ew * ew;
    q2 += q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
  }
  e2 = warp_sum_f(e2);
  q2 = warp_sum_f(q2);
  if (lane == 0) rowstat[n] = make_float2(__fsqrt_ru(e2), __fsqrt_ru(q2));
}

struct RowArgs {
  int64_t N;
  int D, K, L, l;
  int Tc, G, maxs;
  int64_t U;
  int64_t rt0;  // first row tile of the unit range, else 0
  int nslots;   // > 0: every row tile has exactly nslots candidate lists (all-levels kernel)
  const float2 *cand;
  float2 *rowstat;
  float *R;
  __nv_bfloat16 *Rt;
  const void *cb;        // stored codebooks [L,K,D]
  const float *stats;    // this level's RVQ_LEVEL_STATS floats
  int32_t *ids;
  int32_t *fb_list;
  int32_t *fb_count;     // this level's counter
  int32_t *status;
  int last;              // no operand copy needed after the last level
  // register-resident path (D <= 1024)
  const void *src;       // residual before this level: R, or the features at level 0
  int32_t *fb_next;      // next level's fallback counter to clear, or null
  const int64_t *offsets;  // checked at level 0, else null
  int64_t B;
};

// Where a level's input residual comes from.
enum RowSrc { SRC_R = 0, SRC_X_F32 = 1, SRC_X_BF16 = 2 };

template <int SRC>
__device__ __forceinline__ float4 ld_src4(const void *p, int64_t off) {
  if constexpr (SRC == SRC_X_BF16) {
    uint2 raw = __ldg(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p) + off));
    float2 x = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.x));
    float2 y = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.y));
    return make_float4(x.x, x.y, y.x, y.y);
  } else if constexpr (SRC == SRC_X_F32) {
    return __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(p) + off));
  } else {  // the running residual, written by the previous level: read at L2, never a stale L1 line
    return __ldcg(reinterpret_cast<const float4 *>(static_cast<const float *>(p) + off));
  }
}

__device__ __forceinline__ float error_bound(const float *st, float2 rs, int D) {
  const float cmax = st[0], dcmax = st[1], cqmax = st[2], nmax = st[3];
  // fp32 accumulation of D products and the three norm parts (truncation allowed)
  const float gamma = static_cast<float>(D + 32) * 2.384185791015625e-07f;  // (D+32) 2^-22
  // norms: fp32 lane sums of ceil(D/32) squares combined in fp64, then rounded to fp32
  const float norm_err = static_cast<float>(D / 32 + 2) * 5.9604644775390625e-08f;  // (D/32+2) 2^-24
  const float e = norm_err * nmax                                   // n vs ||c||^2
                  + 2.f * (rs.x * cmax + rs.y * dcmax)              // bf16 rounding of r and c
                  + 2.f * gamma * (rs.y * cqmax + 0.51f * nmax)     // tensor-core accumulation
                  + 1.1920928955078125e-07f * nmax;                 // three-part bf16 split of n/2
  return 1.01f * e;
}

// Exact squared distance ||r - c||^2 with fp32 differences widened to fp64 and fp64 sums.
template <bool CB_BF16>
__device__ __forceinline__ double exact_dist(const float *r, const void *cb, int64_t coff, int D, int lane) {
  double s = 0.0;
  for (int i = lane * 4; i < D; i += 128) {
    const float4 v = *reinterpret_cast<const float4 *>(r + i);
    const float4 c = ld4<CB_BF16>(cb, coff + i);
    const double a = static_cast<double>(v.x) - c.x, b = static_cast<double>(v.y) - c.y;
    const double e = static_cast<double>(v.z) - c.z, f = static_cast<double>(v.w) - c.w;
    s += a * a + b * b + e * e + f * f;
  }
  return warp_sum_d(s);
}

// r -= c (fp32), write the ids entry and, unless this was the last level, the next operand row.
template <bool CB_BF16>
__device__ __forceinline__ void accept_row(const RowArgs &a, int64_t n, int id, int lane) {
  float *r = a.R + n * a.D;
  const int64_t coff = (static_cast<int64_t>(a.l) * a.K + id) * a.D;
  for (int i = lane * 4; i < a.D; i += 128) {
    float4 v = *reinterpret_cast<float4 *>(r + i);
    const float4 c = ld4<CB_BF16>(a.cb, coff + i);
    v.x -= c.x;
    v.y -= c.y;
    v.z -= c.z;
    v.w -= c.w;
    *reinterpret_cast<float4 *>(r + i) = v;
  }
  __syncwarp();
  if (!a.last) {
    const float2 st = write_operand_row(r, a.Rt + n * a.D, a.D, lane);
    if (lane == 0) a.rowstat[n] = st;
  }
  if (lane == 0) a.ids[n * a.L + a.l] = id;
}

template <bool CB_BF16>
__global__ void __launch_bounds__(256) rescore_kernel(const RowArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t n = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (n >= a.N) return;
  const int64_t rt = n / BM;
  const int rin = static_cast<int>(n - rt * BM);
  const int64_t ut = rt - a.rt0;  // the unit row tile this 128-row tile belongs to
  const int c0 = cta_of_unit(ut * a.Tc, a.U, a.G);
  const int c1 = cta_of_unit(ut * a.Tc + a.Tc - 1, a.U, a.G);
  const int ncand = (c1 - c0 + 1) * TOPK;

  float dv[CPL];
  int iv[CPL];
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    const int e = lane + 32 * h;
    dv[h] = inf_f();
    iv[h] = -1;
    if (e < ncand) {
      const int slot = e / TOPK, t = e - slot * TOPK;
      const float2 c = __ldcg(a.cand + ((rt * a.maxs + slot) * BM + rin) * TOPK + t);
      dv[h] = c.x;
      iv[h] = __float_as_int(c.y);
    }
  }
  // T: smallest score that some list dropped (a list's last entry; +inf if the list is short)
  float tl = inf_f(), ml = inf_f();
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    const int e = lane + 32 * h;
    if (e < ncand && (e % TOPK) == TOPK - 1) tl = fminf(tl, dv[h]);
    ml = fminf(ml, dv[h]);
  }
  const float T = warp_min_f(tl);
  const float dmin = warp_min_f(ml);
  // + the index bits the chunk-merge path stores in candidate keys (relative change < 2^-18)
  const float E = error_bound(a.stats, a.rowstat[n], a.D) +
                  7.62939453125e-06f * (fabsf(dmin) + (T < 1e30f ? fabsf(T) : 0.f));  // 2^-17

  const float *r = a.R + n * a.D;
  double rr = 0.0;
  for (int i = lane * 4; i < a.D; i += 128) {
    const float4 v = *reinterpret_cast<const float4 *>(r + i);
    rr += static_cast<double>(v.x) * v.x + static_cast<double>(v.y) * v.y + static_cast<double>(v.z) * v.z +
          static_cast<double>(v.w) * v.w;
  }
  rr = warp_sum_d(rr);

  double best = inf_d();
  int best_id = 0x7fffffff;
  const float lim = dmin + 2.f * E;
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    unsigned mask = __ballot_sync(0xffffffffu, iv[h] >= 0 && dv[h] <= lim);
    while (mask) {
      const int src = __ffs(mask) - 1;
      mask &= mask - 1;
      const int id = __shfl_sync(0xffffffffu, iv[h], src);
      const double d = exact_dist<CB_BF16>(r, a.cb, (static_cast<int64_t>(a.l) * a.K + id) * a.D, a.D, lane);
      if (d < best || (d == best && id < best_id)) {
        best = d;
        best_id = id;
      }
    }
  }
  const bool certified = best_id != 0x7fffffff && (best - rr) < (static_cast<double>(T) - static_cast<double>(E));
  if (!certified) {
    if (lane == 0) {
      const int pos = atomicAdd(a.fb_count, 1);
      a.fb_list[pos] = static_cast<int32_t>(n);
    }
    return;
  }
  accept_row<CB_BF16>(a, n, best_id, lane);
}

// Exact scan of all K codewords for the queued rows of this level.
template <bool CB_BF16>
__global__ void __launch_bounds__(256) fallback_kernel(const RowArgs a) {
  extern __shared__ double sr[];  // residual row widened to fp64
  __shared__ double wbest[8];
  __shared__ int wid[8];
  __shared__ int chosen;
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int count = *a.fb_count;
  for (int j = blockIdx.x; j < count; j += gridDim.x) {
    const int64_t n = a.fb_list[j];
    const float *r = a.R + n * a.D;
    __syncthreads();
    for (int i = threadIdx.x; i < a.D; i += blockDim.x) sr[i] = static_cast<double>(r[i]);
    __syncthreads();
    double bd = inf_d();
    int bk = 0x7fffffff;
    for (int k = warp; k < a.K; k += 8) {
      const int64_t coff = (static_cast<int64_t>(a.l) * a.K + k) * a.D;
      double s = 0.0;
      if constexpr (CB_BF16) {
        const __nv_bfloat16 *c = static_cast<const __nv_bfloat16 *>(a.cb) + coff;
        for (int i = lane; i < a.D; i += 32) {
          const double t = sr[i] - static_cast<double>(__bfloat162float(c[i]));
          s += t * t;
        }
      } else {
        const float *c = static_cast<const float *>(a.cb) + coff;
        for (int i = lane; i < a.D; i += 32) {
          const double t = sr[i] - static_cast<double>(__ldg(c + i));
          s += t * t;
        }
      }
      s = warp_sum_d(s);
      if (s < bd) {
        bd = s;
        bk = k;
      }
    }
    if (lane == 0) {
      wbest[warp] = bd;
      wid[warp] = bk;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double b = wbest[0];
      int k = wid[0];
      for (int w = 1; w < 8; ++w)
        if (wbest[w] < b || (wbest[w] == b && wid[w] < k)) {
          b = wbest[w];
          k = wid[w];
        }
      chosen = k;
    }
    __syncthreads();
    if (warp == 0) {
      if (chosen >= 0 && chosen < a.K) {
        accept_row<CB_BF16>(a, n, chosen, lane);
      } else if (lane == 0) {  // only reachable with non-finite inputs
        a.ids[n * a.L + a.l] = -1;
        set_status(a.status, RVQ_ERR_ARG);
      }
    }
  }
}

// ---------------------------------------------------------------- register-resident row kernels
// One warp per row with the whole residual row in registers (NCH float4 per lane, D <= 128*NCH):
// the candidate lists, the row and the winner's codeword are each read once, and the updated
// residual, its bf16 operand copy and row statistics are written from registers.

// Packed-batch bookkeeping: offsets[0] = 0, non-decreasing, offsets[B] = N (checked, not used).
__device__ __forceinline__ void check_offsets(const RowArgs &a, int64_t gtid, int64_t nthreads) {
  for (int64_t b = gtid; b < a.B; b += nthreads)
    if (a.offsets[b] > a.offsets[b + 1]) set_status(a.status, RVQ_ERR_ARG);
  if (gtid == 0 && (a.offsets[0] != 0 || a.offsets[a.B] != a.N)) set_status(a.status, RVQ_ERR_ARG);
}

// r -= c for a register-resident row (element lane*4 + 128k of chunk k), then the ids entry and,
// unless this was the last level, the next level's bf16 operand row and its rounding statistics.
template <int NCH>
__device__ __forceinline__ void apply_row(const RowArgs &a, int64_t n, const float4 (&rv)[NCH],
                                          const float4 (&c)[NCH], int id, int lane) {
  float e2 = 0.f, q2 = 0.f;
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int i = lane * 4 + k * 128;
    if (i >= a.D) break;
    float4 v = rv[k];
    v.x -= c[k].x;
    v.y -= c[k].y;
    v.z -= c[k].z;
    v.w -= c[k].w;
    *reinterpret_cast<float4 *>(a.R + n * a.D + i) = v;
    if (!a.last) {
      float4 q;
      store_bf16x4(a.Rt + n * a.D + i, v, &q);
      const float ex = v.x - q.x, ey = v.y - q.y, ez = v.z - q.z, ew = v.w - q.w;
      e2 += ex * ex + ey * ey + ez * ez + ew * ew;
      q2 += q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
    }
  }
  if (!a.last) {
    e2 = warp_sum_f(e2);
    q2 = warp_sum_f(q2);
    if (lane == 0) a.rowstat[n] = make_float2(__fsqrt_ru(e2), __fsqrt_ru(q2));
  }
  if (lane == 0) a.ids[n * a.L + a.l] = id;
}

// Certificate, exact rescore when needed, and the residual update of row n (one warp).  Returns
// whether the row was settled; an uncertified row is appended to a.fb_list when that is set.
template <bool CB_BF16, int SRC, int NCH>
__device__ __forceinline__ bool rescore_row(const RowArgs &a, int64_t n, int lane) {
  const int64_t rt = n / BM;
  const int rin = static_cast<int>(n - rt * BM);
  int ncand = a.nslots * TOPK;
  if (a.nslots <= 0) {
    const int64_t ut = rt - a.rt0;
    const int c0 = cta_of_unit(ut * a.Tc, a.U, a.G);
    const int c1 = cta_of_unit(ut * a.Tc + a.Tc - 1, a.U, a.G);
    ncand = (c1 - c0 + 1) * TOPK;
  }

  // independent loads first: the residual row and the candidate lists
  float4 rv[NCH];
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int i = lane * 4 + k * 128;
    rv[k] = i < a.D ? ld_src4<SRC>(a.src, n * a.D + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float dv[CPL];
  int iv[CPL];
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    const int e = lane + 32 * h;
    dv[h] = inf_f();
    iv[h] = -1;
    if (e < ncand) {
      const int slot = e / TOPK, t = e - slot * TOPK;
      const float2 c = __ldcg(a.cand + ((rt * a.maxs + slot) * BM + rin) * TOPK + t);
      dv[h] = c.x;
      iv[h] = __float_as_int(c.y);
    }
  }
  float2 rs = make_float2(0.f, 0.f);
  if constexpr (SRC != SRC_X_BF16) rs = __ldcg(a.rowstat + n);

  // r is its own bf16 copy when it comes straight from bf16 features: e_r = 0, ||r~|| = ||r||
  if constexpr (SRC == SRC_X_BF16) {
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < NCH; ++k) q += rv[k].x * rv[k].x + rv[k].y * rv[k].y + rv[k].z * rv[k].z + rv[k].w * rv[k].w;
    rs = make_float2(0.f, __fsqrt_ru(1.0001f * warp_sum_f(q)));
  }

  float tl = inf_f(), ml = inf_f();
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    const int e = lane + 32 * h;
    if (e < ncand && (e % TOPK) == TOPK - 1) tl = fminf(tl, dv[h]);
    ml = fminf(ml, dv[h]);
  }
  const float T = warp_min_f(tl);
  const float dmin = warp_min_f(ml);
  const float E = error_bound(a.stats, rs, a.D) + 7.62939453125e-06f * (fabsf(dmin) + (T < 1e30f ? fabsf(T) : 0.f));
  const float lim = dmin + 2.f * E;
  unsigned pm[CPL];
  int nplaus = 0;
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    pm[h] = __ballot_sync(0xffffffffu, iv[h] >= 0 && dv[h] <= lim);
    nplaus += __popc(pm[h]);
  }

  int best_id = 0x7fffffff;
  float4 cbest[NCH];
  if (nplaus == 1 && T - dmin > 2.f * E) {
    // One candidate within 2E of the best score and every dropped score more than 2E above it:
    // its true distance is below every other codeword's, so no exact rescore is needed.
#pragma unroll
    for (int h = 0; h < CPL; ++h)
      if (pm[h]) best_id = __shfl_sync(0xffffffffu, iv[h], __ffs(pm[h]) - 1);
    const int64_t coff = (static_cast<int64_t>(a.l) * a.K + best_id) * a.D;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int i = lane * 4 + k * 128;
      cbest[k] = i < a.D ? ld4<CB_BF16>(a.cb, coff + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else {
    double rr = 0.0;
#pragma unroll
    for (int k = 0; k < NCH; ++k)
      rr += static_cast<double>(rv[k].x) * rv[k].x + static_cast<double>(rv[k].y) * rv[k].y +
            static_cast<double>(rv[k].z) * rv[k].z + static_cast<double>(rv[k].w) * rv[k].w;
    rr = warp_sum_d(rr);
    double best = inf_d();
#pragma unroll
    for (int h = 0; h < CPL; ++h) {
      unsigned mask = pm[h];
      while (mask) {
        const int srcl = __ffs(mask) - 1;
        mask &= mask - 1;
        const int id = __shfl_sync(0xffffffffu, iv[h], srcl);
        const int64_t coff = (static_cast<int64_t>(a.l) * a.K + id) * a.D;
        float4 c[NCH];
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
          const int i = lane * 4 + k * 128;
          c[k] = i < a.D ? ld4<CB_BF16>(a.cb, coff + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        double dd = 0.0;
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
          const double e0 = static_cast<double>(rv[k].x) - c[k].x, e1 = static_cast<double>(rv[k].y) - c[k].y;
          const double e2 = static_cast<double>(rv[k].z) - c[k].z, e3 = static_cast<double>(rv[k].w) - c[k].w;
          dd += e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
        }
        dd = warp_sum_d(dd);
        if (dd < best || (dd == best && id < best_id)) {
          best = dd;
          best_id = id;
        }
      }
    }
    const bool certified =
        best_id != 0x7fffffff && (best - rr) < (static_cast<double>(T) - static_cast<double>(E));
    if (!certified) {
      if (a.fb_list && lane == 0) {
        const int pos = atomicAdd(a.fb_count, 1);
        a.fb_list[pos] = static_cast<int32_t>(n);
      }
      return false;
    }
    // the winner's row again (cheaper than keeping the best candidate row live in registers)
    const int64_t coff = (static_cast<int64_t>(a.l) * a.K + best_id) * a.D;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int i = lane * 4 + k * 128;
      cbest[k] = i < a.D ? ld4<CB_BF16>(a.cb, coff + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  apply_row<NCH>(a, n, rv, cbest, best_id, lane);
  return true;
}

template <bool CB_BF16, int SRC, int NCH>
__global__ void __launch_bounds__(256, 2) rescore_fast_kernel(const RowArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gtid == 0 && a.fb_next) *a.fb_next = 0;
  if (a.offsets) check_offsets(a, gtid, static_cast<int64_t>(gridDim.x) * blockDim.x);
  const int64_t n = gtid >> 5;
  if (n >= a.N) return;
  rescore_row<CB_BF16, SRC, NCH>(a, n, lane);
}

// Exact scan of all K codewords for one queued row (all warps of the block; sr holds D doubles,
// wbest/wid one slot per warp).  The chosen codeword is applied like an accepted rescore.
template <bool CB_BF16, int SRC>
__device__ __forceinline__ void fallback_row(const RowArgs &a, int64_t n, double *sr, double *wbest, int *wid,
                                             int *chosen) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  __syncthreads();
  for (int i = threadIdx.x * 4; i < a.D; i += blockDim.x * 4) {
    const float4 v = ld_src4<SRC>(a.src, n * a.D + i);
    sr[i] = v.x;
    sr[i + 1] = v.y;
    sr[i + 2] = v.z;
    sr[i + 3] = v.w;
  }
  __syncthreads();
  double bd = inf_d();
  int bk = 0x7fffffff;
  for (int k = warp; k < a.K; k += nwarps) {
    const int64_t coff = (static_cast<int64_t>(a.l) * a.K + k) * a.D;
    double acc = 0.0;
    for (int i = lane * 4; i < a.D; i += 128) {
      const float4 c = ld4<CB_BF16>(a.cb, coff + i);
      const double e0 = sr[i] - c.x, e1 = sr[i + 1] - c.y, e2 = sr[i + 2] - c.z, e3 = sr[i + 3] - c.w;
      acc += e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
    }
    acc = warp_sum_d(acc);
    if (acc < bd) {
      bd = acc;
      bk = k;
    }
  }
  if (lane == 0) {
    wbest[warp] = bd;
    wid[warp] = bk;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double b = wbest[0];
    int k = wid[0];
    for (int w = 1; w < nwarps; ++w)
      if (wbest[w] < b || (wbest[w] == b && wid[w] < k)) {
        b = wbest[w];
        k = wid[w];
      }
    *chosen = k;
  }
  __syncthreads();
  if (warp == 0) {
    const int id = *chosen;
    if (id < 0 || id >= a.K) {  // only reachable with non-finite inputs
      if (lane == 0) {
        a.ids[n * a.L + a.l] = -1;
        set_status(a.status, RVQ_ERR_ARG);
      }
      return;
    }
    const int64_t coff = (static_cast<int64_t>(a.l) * a.K + id) * a.D;
    float e2 = 0.f, q2 = 0.f;
    for (int i = lane * 4; i < a.D; i += 128) {
      const float4 c = ld4<CB_BF16>(a.cb, coff + i);
      const float4 v = make_float4(static_cast<float>(sr[i]) - c.x, static_cast<float>(sr[i + 1]) - c.y,
                                   static_cast<float>(sr[i + 2]) - c.z, static_cast<float>(sr[i + 3]) - c.w);
      *reinterpret_cast<float4 *>(a.R + n * a.D + i) = v;
      if (!a.last) {
        float4 q;
        store_bf16x4(a.Rt + n * a.D + i, v, &q);
        const float ex = v.x - q.x, ey = v.y - q.y, ez = v.z - q.z, ew = v.w - q.w;
        e2 += ex * ex + ey * ey + ez * ez + ew * ew;
        q2 += q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
      }
    }
    if (!a.last) {
      e2 = warp_sum_f(e2);
      q2 = warp_sum_f(q2);
      if (lane == 0) a.rowstat[n] = make_float2(__fsqrt_ru(e2), __fsqrt_ru(q2));
    }
    if (lane == 0) a.ids[n * a.L + a.l] = id;
  }
}

// Exact scan of all K codewords for the rows this level's rescore could not certify.
template <bool CB_BF16, int SRC>
__global__ void __launch_bounds__(256) fallback_fast_kernel(const RowArgs a) {
  extern __shared__ double sr[];  // residual row widened to fp64
  __shared__ double wbest[8];
  __shared__ int wid[8];
  __shared__ int chosen;
  griddep_launch_dependents();
  griddep_wait();
  const int count = *a.fb_count;
  for (int j = blockIdx.x; j < count; j += gridDim.x) fallback_row<CB_BF16, SRC>(a, a.fb_list[j], sr, wbest, wid, &chosen);
}

template <bool CB_BF16, int SRC>
inline cudaError_t launch_rows_fast(const RowArgs &ra, int nch, unsigned row_blocks, int fb_blocks, size_t fb_smem,
                                    cudaStream_t s) {
  cudaError_t e;
  switch (nch) {
    case 1: e = launch_pdl(rescore_fast_kernel<CB_BF16, SRC, 1>, dim3(row_blocks), dim3(256), 0, s, ra); break;
    case 2: e = launch_pdl(rescore_fast_kernel<CB_BF16, SRC, 2>, dim3(row_blocks), dim3(256), 0, s, ra); break;
    case 4: e = launch_pdl(rescore_fast_kernel<CB_BF16, SRC, 4>, dim3(row_blocks), dim3(256), 0, s, ra); break;
    default: e = launch_pdl(rescore_fast_kernel<CB_BF16, SRC, 8>, dim3(row_blocks), dim3(256), 0, s, ra); break;
  }
  if (e != cudaSuccess) return e;
  return launch_pdl(fallback_fast_kernel<CB_BF16, SRC>, dim3(fb_blocks), dim3(256), fb_smem, s, ra);
}

// ---------------------------------------------------------------- all levels in one launch
// One launch with every CTA resident runs every level as a dataflow over row tiles:
//
//  * GEMM chunks.  Chunk (l, rt, j) scores row tile rt against codeword tiles [jS, (j+1)S) of
//    level l and writes one partial top-8 list per row into slot j.  Chunks are numbered level by
//    level, row tile by row tile, and CTA c takes chunks c, c+G, c+2G, ... (CTA pairs: pair c
//    takes the chunks of 256-row units, each CTA scoring its own row tile of the unit).  The TMA
//    producer, MMA issuer, norm splitter and epilogue warps walk that sequence with the
//    shared-memory ring, the TMEM buffers and the mbarrier phases carried from chunk to chunk.
//    Before loading chunk (l, rt, j) the producer waits until row tile rt is settled at level l-1.
//  * Certificate tasks.  RW warps per CTA take tasks (l, rt, g) the same way (RPT rows each):
//    once all NC chunks of (l, rt) are written they certify the rows, apply r -= C_l[id] and
//    count the settled rows.  A row the certificate cannot settle goes to a queue whose exact
//    scan is split into NS codeword slices that any certificate warp picks up while it would
//    otherwise wait; the warp finishing a row's last slice reduces the slices, applies the winner
//    and counts the row.
//
// Counters (zeroed by the host, all acquire/release at GPU scope):
//   chunk_done[l][rt]  group-0 epilogue warps through a chunk of (l, rt)   (complete at 4 NC)
//   cert_done[l][rt]   settled rows of (l, rt)                             (complete at the rows)
// so level l+1 of a row tile starts while later row tiles of level l are still being scored,
// and the certificate work runs under the tensor-core work.  Every wait is bounded: it gives up
// when neither its counter nor the grid's progress word has moved for two seconds.
// Epilogue and certificate warps of the all-levels kernel, after the three GEMM-role warps.
// D in (512, 1024]: 4 epilogue + 5 more warps (12 per block).  Measured against 8 + 5 (16 warps)
// with clocks sampled: packed (65503 rows) 1249 vs 1223 TFLOP/s at 1965 MHz, detok (262144 rows)
// 883 vs 852 TFLOP/s per GHz under the power cap, image unchanged; 4 epilogue + 9 certificate
// warps in 16 was 9% slower on image.  D in (128, 256]: 8 + 5 (16 warps).
constexpr int FLOW_EPI_WIDE = 4;
constexpr int FLOW_RW_WIDE = 5;
constexpr int FLOW_EPI_NARROW = 8;
constexpr int FLOW_RW_NARROW = 5;
// Idle warps among the five (bit i = warp CERT0 + i; warp w runs on SM sub-partition w mod 4): the
// one that would share the MMA issuer's sub-partition (4 certificate warps; with 8 epilogue warps
// at D = 1024 image ran 13.2 vs 13.1 Mtok/s with 5, 12.8 with 3); at D = 256 also the TMA
// producer's (3 certificate warps; offline 7.61 vs 7.45 with 4).
constexpr int FLOW_SKIP_WIDE = 0b00100;
constexpr int FLOW_SKIP_NARROW = 0b00110;
constexpr int EXACT_QCAP = 1024;   // queued rows whose exact scan is split into slices
constexpr int EXACT_NS_MAX = 256;  // codeword slices per queued row

struct FlowArgs {
  int L;
  int64_t RT;
  int NC, S;        // chunks per row tile, codeword tiles per chunk
  int RPT;          // rows per certificate task (divides 128)
  int NS, slice;    // exact-scan slices per queued row, codewords per slice
  uint32_t *chunk_done;  // [L, RT]
  uint32_t *cert_done;   // [L, RT]
  uint32_t *ctr;         // queued rows, next slice, settled rows, progress
  int4 *ex_entry;        // [EXACT_QCAP]: row, level, ready flag, slices done
  double2 *ex_part;      // [EXACT_QCAP, NS]: best distance of a slice, its codeword id
  int32_t *fb_level;     // [L] rows per level that took the exact scan
  const float *norms;    // [L, K]
  const float *level_stats;
};

// Publish this warp's global writes and add v (warp-uniform) to *ctr.  TMA: the writes are also
// made visible to the async proxy (later TMA loads of the residual operand).
template <bool TMA>
__device__ __forceinline__ void warp_release_add(uint32_t *ctr, uint32_t v, int lane) {
  if constexpr (TMA) fence_proxy_async_global();
  __syncwarp();
  if (lane == 0 && v) red_release_add_gpu(ctr, v);
}

// Exact scan of all K codewords of level a.l for row n by one warp (slow path, used only when
// the slice queue is full): lane j scores codewords j, j+32, ... with fp64 accumulation of fp32
// differences, the residual row broadcast from the registers that hold it; lowest index on
// ties.  Applies the winner like an accepted rescore.
template <bool CB_BF16, int SRC, int NCH>
__device__ __noinline__ void exact_row(const RowArgs &a, int64_t n, int lane) {
  float4 rv[NCH];
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int i = lane * 4 + k * 128;
    rv[k] = i < a.D ? ld_src4<SRC>(a.src, n * a.D + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int64_t lvl = static_cast<int64_t>(a.l) * a.K;
  double best = inf_d();
  int bid = 0x7fffffff;
  for (int k0 = 0; k0 < a.K; k0 += 32) {
    const int k = k0 + lane;
    const int64_t coff = (lvl + (k < a.K ? k : a.K - 1)) * a.D;
    double acc = 0.0;
#pragma unroll
    for (int q = 0; q < NCH; ++q) {
#pragma unroll 4
      for (int s = 0; s < 32; ++s) {
        if (q * 128 + s * 4 >= a.D) break;
        const float rx = __shfl_sync(0xffffffffu, rv[q].x, s), ry = __shfl_sync(0xffffffffu, rv[q].y, s);
        const float rz = __shfl_sync(0xffffffffu, rv[q].z, s), rw = __shfl_sync(0xffffffffu, rv[q].w, s);
        const float4 c = ld4<CB_BF16>(a.cb, coff + q * 128 + s * 4);
        const double e0 = static_cast<double>(rx) - c.x, e1 = static_cast<double>(ry) - c.y;
        const double e2 = static_cast<double>(rz) - c.z, e3 = static_cast<double>(rw) - c.w;
        acc += e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
      }
    }
    if (k < a.K && acc < best) {
      best = acc;
      bid = k;
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bid, off);
    if (ob < best || (ob == best && oi < bid)) {
      best = ob;
      bid = oi;
    }
  }
  if (bid < 0 || bid >= a.K) {  // only reachable with non-finite inputs
    if (lane == 0) {
      a.ids[n * a.L + a.l] = -1;
      set_status(a.status, RVQ_ERR_ARG);
    }
    return;
  }
  float4 c[NCH];
  const int64_t coff = (lvl + bid) * a.D;
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int i = lane * 4 + k * 128;
    c[k] = i < a.D ? ld4<CB_BF16>(a.cb, coff + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  apply_row<NCH>(a, n, rv, c, bid, lane);
}

// One slice of a queued row's exact scan: codewords [k0, k1) of level a.l, one codeword per
// warp step (coalesced rows), UNR codewords in flight; fp64 accumulation of fp32 differences,
// lowest index on ties.  Returns the slice's best distance and codeword in every lane.
template <bool CB_BF16, int NCH>
__device__ __forceinline__ void exact_slice(const RowArgs &a, int64_t n, int k0, int k1, const float4 (&rv)[NCH],
                                            int lane, double &best, int &bid) {
  constexpr int UNR = NCH <= 2 ? 4 : NCH <= 4 ? 2 : 1;
  const int64_t lvl = static_cast<int64_t>(a.l) * a.K;
  best = inf_d();
  bid = 0x7fffffff;
  for (int k = k0; k < k1; k += UNR) {
    double acc[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int kk = k + u < k1 ? k + u : k1 - 1;
      const int64_t coff = (lvl + kk) * a.D;
      float4 c[NCH];
#pragma unroll
      for (int q = 0; q < NCH; ++q) {
        const int i = lane * 4 + q * 128;
        c[q] = i < a.D ? ld4<CB_BF16>(a.cb, coff + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      double s = 0.0;
#pragma unroll
      for (int q = 0; q < NCH; ++q) {
        const double e0 = static_cast<double>(rv[q].x) - c[q].x, e1 = static_cast<double>(rv[q].y) - c[q].y;
        const double e2 = static_cast<double>(rv[q].z) - c[q].z, e3 = static_cast<double>(rv[q].w) - c[q].w;
        s += e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
      }
      acc[u] = s;
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const double d = warp_sum_d(acc[u]);
      if (k + u < k1 && d < best) {
        best = d;
        bid = k + u;
      }
    }
  }
}

// RW warps follow the GEMM roles; those in the bit mask SKIP (relative to CERT0) stay idle, so that
// no certificate work shares a scheduler sub-partition (warp w runs on sub-partition w % 4) with
// the MMA issuer or, when set, the TMA producer.
template <int EPI, int RW, int SKIP>
struct FlowCfg {
  static constexpr int THREADS = GemmCfg<EPI>::THREADS + RW * 32;
  static constexpr int CERT0 = EPI + 3;  // first of the RW warps after the GEMM roles
  static constexpr int CERT_WARPS = RW - __builtin_popcount(SKIP);
};

// Shared memory of the all-levels kernel.  A CTA of a pair (cta_group::2) loads its own 128 rows
// and half of each 256-codeword tile, so a stage is A 16 KB + B 16 KB and six stages fit where
// four single-CTA stages of 48 KB do.
template <int EPI, bool PAIR>
struct FlowMem : GemmCfg<EPI> {
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // codeword rows of a tile this CTA loads
  static constexpr int STAGE = A_BYTES + B_ROWS * BK * 2;
  static constexpr int NSTAGE = PAIR ? 6 : GemmCfg<EPI>::NSTAGE;
  static constexpr int AUG_A_OFF = NSTAGE * STAGE;
  static constexpr int AUG_B_OFF = AUG_A_OFF + AUG_A_BYTES;
  static constexpr int MERGE_OFF = AUG_B_OFF + 2 * AUG_B_BYTES;
  static constexpr int BAR_OFF = MERGE_OFF + (GemmCfg<EPI>::GROUPS - 1) * BM * TOPK * 8;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;
  static_assert(SMEM <= 232448, "dynamic shared memory above the 227 KB per-block limit");
  static_assert(!PAIR || GemmCfg<EPI>::GROUPS == 1, "pairs run one epilogue column group");
};

template <int EPI, int RW, int SKIP, bool CB_BF16, bool X_BF16, int NCH, bool PAIR>
__global__ void __launch_bounds__(FlowCfg<EPI, RW, SKIP>::THREADS, 1)
    encode_flow_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB3, const GemmArgs a, const RowArgs r0,
                       const FlowArgs fa) {
  using C = FlowMem<EPI, PAIR>;
  constexpr int NSTAGE = C::NSTAGE;
  constexpr int CERT0 = FlowCfg<EPI, RW, SKIP>::CERT0;
  constexpr int CW = FlowCfg<EPI, RW, SKIP>::CERT_WARPS;
  constexpr int SRC0 = X_BF16 ? SRC_X_BF16 : SRC_X_F32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *aug_a = smem + C::AUG_A_OFF;
  uint8_t *aug_b = smem + C::AUG_B_OFF;
  float2 *mbuf = reinterpret_cast<float2 *>(smem + C::MERGE_OFF);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
  uint64_t *empty = full + NSTAGE;
  uint64_t *tfull = empty + NSTAGE;
  uint64_t *tempty = tfull + 2;
  uint64_t *afull = tempty + 2;
  uint64_t *mready = afull + 2;
  uint64_t *mdone = mready + 1;
  uint64_t *mma_done = mdone + 1;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  volatile int *never = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = a.D / BK;
  const uint32_t G = gridDim.x;
  const int64_t RT = fa.RT;
  // Chunks are walked by CTAs, or by CTA pairs over 256-row units (unit u holds row tiles 2u and
  // 2u+1, the second of which may lie past the last row tile).
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0: the pair's leader (issues the MMAs)
  const uint32_t GW = PAIR ? G / 2 : G;                  // chunk walkers
  const uint32_t wid = PAIR ? blockIdx.x / 2 : blockIdx.x;
  const int64_t RU = PAIR ? (RT + 1) / 2 : RT;           // row units
  const int64_t total_chunks = static_cast<int64_t>(fa.L) * RU * fa.NC;
  auto own_tile = [&](int64_t ru) -> int64_t { return PAIR ? 2 * ru + rank : ru; };
  uint32_t *ex_rows = fa.ctr;
  uint32_t *ex_next = fa.ctr + 1;
  uint32_t *settled = fa.ctr + 2;
  uint32_t *progress = fa.ctr + 3;
  // rows of row tile rt (the last tile may be short)
  auto tile_rows = [&](int64_t rt) -> uint32_t {
    return static_cast<uint32_t>(min(static_cast<int64_t>(BM), a.N - rt * BM));
  };
  // First codeword tile this CTA visits in a chunk of cnt tiles: CTAs spread their starting
  // points over the chunk so they do not all stream the same codeword tile at the same time.
  auto chunk_rot = [&](int cnt) -> int { return static_cast<int>((static_cast<int64_t>(wid) * cnt) / GW); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], (PAIR ? 2 : 1) * C::EPI_THREADS);  // a pair's epilogues both release the leader's
      mbar_init(&afull[b], PAIR ? 64 : 32);
    }
    mbar_init(mready, C::EPI_THREADS - 128 > 0 ? C::EPI_THREADS - 128 : 1);
    mbar_init(mdone, 128);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    *never = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < (AUG_A_BYTES + 2 * AUG_B_BYTES) / 16; i += blockDim.x) {
    uint4 v = make_uint4(0, 0, 0, 0);
    if (i < AUG_A_BYTES / 16 && ((i * 16) % 256) < 128)
      v = make_uint4(BF16_ONE | (static_cast<uint32_t>(BF16_ONE) << 16), BF16_ONE, 0, 0);
    reinterpret_cast<uint4 *>(aug_a)[i] = v;
  }
  fence_proxy_async_smem();
  if (warp == C::ISSUER) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_holder, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // the leader's barriers, as seen from either CTA of a pair
  const uint32_t full_l = PAIR ? mapa_shared(smem_u32(full), 0) : 0u;
  const uint32_t tempty_l = PAIR ? mapa_shared(smem_u32(tempty), 0) : 0u;
  const uint32_t afull_l = PAIR ? mapa_shared(smem_u32(afull), 0) : 0u;

  int p_s = 0;  // producer ring position, kept for the teardown
  uint32_t p_ph = 0;
  int64_t p_issued = 0;

  if (warp == C::PRODUCER) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA0);
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB3);
      bool ok = true;
      for (int64_t t = wid; t < total_chunks && ok; t += GW) {
        const int j = static_cast<int>(t % fa.NC);
        const int64_t rt = own_tile((t / fa.NC) % RU);
        const int l = static_cast<int>(t / (fa.NC * RU));
        if (l > 0 && rt < RT) {  // a pair's second tile past the last row tile holds no rows
          if (!wait_count(fa.cert_done + (l - 1) * RT + rt, tile_rows(rt), progress, abort_flag)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();  // residual rows written by the generic proxy, read by TMA
        }
        const CUtensorMap *mA = l == 0 ? &tmA0 : &tmA;
        const int ct0 = j * fa.S, cnt = min(a.Tc, ct0 + fa.S) - ct0;
        const int rot = chunk_rot(cnt);
        for (int k = 0; k < cnt && ok; ++k) {
          const int ct = ct0 + (rot + k) % cnt;
          for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&empty[p_s], p_ph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t *sa = smem + p_s * C::STAGE;
            if constexpr (PAIR) {  // both CTAs' bytes complete the leader's barrier
              if (rank == 0) mbar_arrive_expect_tx(&full[p_s], 2 * C::STAGE);
              tma_load_2d_pair(mA, full_l + p_s * 8, sa, kb * BK, static_cast<int32_t>(rt * BM));
              tma_load_3d_pair(&tmB3, full_l + p_s * 8, sa + A_BYTES, kb * BK,
                               ct * BN + static_cast<int32_t>(rank) * C::B_ROWS, l);
            } else {
              mbar_arrive_expect_tx(&full[p_s], C::STAGE);
              tma_load_2d(mA, &full[p_s], sa, kb * BK, static_cast<int32_t>(rt * BM));
              tma_load_3d(&tmB3, &full[p_s], sa + A_BYTES, kb * BK, ct * BN, l);
            }
            ++p_issued;
            if (++p_s == NSTAGE) {
              p_s = 0;
              p_ph ^= 1u;
            }
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(a.status, RVQ_ERR_TIMEOUT);
      }
    }
  } else if (warp == C::SPLITTER) {
    // ------------------------------------------------------------ norm split -> B_aug tiles
    int64_t i = 0;
    bool ok = true;
    // this CTA's codeword rows of a tile in groups of 8 (a pair's CTA holds half the tile)
    const bool writer = lane < C::B_ROWS / 8;
    for (int64_t t = wid; t < total_chunks && ok; t += GW) {
      const int j = static_cast<int>(t % fa.NC);
      const int l = static_cast<int>(t / (fa.NC * RU));
      const float *norms_l = fa.norms + static_cast<int64_t>(l) * a.K;
      const int ct0 = j * fa.S, cnt = min(a.Tc, ct0 + fa.S) - ct0;
      const int rot = chunk_rot(cnt);
      for (int k = 0; k < cnt; ++k, ++i) {
        const int ct = ct0 + (rot + k) % cnt;
        const int slot = static_cast<int>(i & 1);
        const int c0 = ct * BN + static_cast<int>(rank) * C::B_ROWS + lane * 8;
        float hv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) hv[q] = (writer && c0 + q < a.K) ? 0.5f * __ldg(norms_l + c0 + q) : 0.f;
        bool got = i < 2 || mbar_wait(&tfull[slot], static_cast<uint32_t>(((i >> 1) - 1) & 1), abort_flag);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(aug_b + slot * AUG_B_BYTES + lane * 128);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (!writer) break;
          uint16_t h1, h2 = 0, h3 = 0;
          if (c0 + q < a.K) {
            h1 = bf16_bits_rn(hv[q]);
            const float r1 = hv[q] - bf16_bits_to_float(h1);
            h2 = bf16_bits_rn(r1);
            const float r2 = r1 - bf16_bits_to_float(h2);
            h3 = bf16_bits_rn(r2);
          } else {
            h1 = BF16_BIG;
          }
          dst[q] = make_uint4(h1 | (static_cast<uint32_t>(h2) << 16), h3, 0, 0);
        }
        fence_proxy_async_smem();
        if constexpr (PAIR)
          mbar_arrive_cluster(afull_l + slot * 8);
        else
          mbar_arrive(&afull[slot]);
      }
    }
    if (!ok) {
      *abort_flag = 1;
      set_status(a.status, RVQ_ERR_TIMEOUT);
    }
  } else if (warp == C::ISSUER) {
    // ------------------------------------------------------------ MMA issuer (a pair's leader)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc_main = idesc_bf16_f32(PAIR ? 2 * BM : BM, BN, true);
      constexpr uint32_t idesc_aug = idesc_bf16_f32(PAIR ? 2 * BM : BM, BN, false);
      const uint64_t adesc_aug = sdesc_k_noswizzle(smem_u32(aug_a), 128, 256);
      int m_s = 0;
      uint32_t m_ph = 0;
      int64_t i = 0;
      bool ok = true;
      for (int64_t t = wid; t < total_chunks && ok; t += GW) {
        const int j = static_cast<int>(t % fa.NC);
        const int cnt = min(a.Tc, j * fa.S + fa.S) - j * fa.S;
        for (int k = 0; k < cnt && ok; ++k, ++i) {
          const int buf = static_cast<int>(i & 1);
          const uint32_t tph = static_cast<uint32_t>((i >> 1) & 1);
          if (!mbar_wait(&tempty[buf], tph ^ 1u, abort_flag) || !mbar_wait(&afull[buf], tph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tmem_base + static_cast<uint32_t>(buf * BN);
          const uint64_t bdesc_aug = sdesc_k_noswizzle(smem_u32(aug_b + buf * AUG_B_BYTES), 128, 128);
          if constexpr (PAIR)
            umma_f16_pair(dt, adesc_aug, bdesc_aug, idesc_aug, 0u);
          else
            umma_f16(dt, adesc_aug, bdesc_aug, idesc_aug, 0u);
          for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&full[m_s], m_ph, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + m_s * C::STAGE);
            const uint64_t ad = sdesc_k128(sa);
            const uint64_t bd = sdesc_k128(sa + A_BYTES);
#pragma unroll
            for (int k = 0; k < BK / UK; ++k) {
              const uint64_t step = static_cast<uint64_t>(k * UK * 2 / 16);
              if constexpr (PAIR)
                umma_f16_pair(dt, ad + step, bd + step, idesc_main, 1u);
              else
                umma_f16(dt, ad + step, bd + step, idesc_main, 1u);
            }
            if constexpr (PAIR)
              umma_commit_pair_both(&empty[m_s]);  // frees the stage in both CTAs
            else
              umma_commit(&empty[m_s]);
            if (++m_s == NSTAGE) {
              m_s = 0;
              m_ph ^= 1u;
            }
          }
          if (!ok) break;
          if constexpr (PAIR)
            umma_commit_pair_both(&tfull[buf]);  // both CTAs' epilogues may read their TMEM rows
          else
            umma_commit(&tfull[buf]);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(a.status, RVQ_ERR_TIMEOUT);
      }
    }
  } else if (warp < EPI) {
    // ------------------------------------------------------------ epilogue: running top-8 per chunk
    const int quad = warp & 3;
    const int grp = warp >> 2;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    float bd[TOPK];
    int bi[TOPK];
    int64_t i = 0;
    uint32_t nflush = 0;
    bool ok = true;
    for (int64_t t = wid; t < total_chunks && ok; t += GW) {
      const int j = static_cast<int>(t % fa.NC);
      const int64_t rt = own_tile((t / fa.NC) % RU);
      const bool rows_here = rt < RT;  // false only for a pair's second tile past the last row tile
      const int l = static_cast<int>(t / (fa.NC * RU));
#pragma unroll
      for (int q = 0; q < TOPK; ++q) {
        bd[q] = inf_f();
        bi[q] = -1;
      }
      // slot j of (l-1, rt) must have been read by every certificate task before it is rewritten:
      // the producer already waited for that, so this load (checked at the flush) only orders it
      uint32_t settled_prev = 0xffffffffu;
      if (grp == 0 && lane == 0 && l > 0 && rows_here)
        settled_prev = ld_acquire_gpu(fa.cert_done + (l - 1) * RT + rt);
      const int ct0 = j * fa.S, cnt = min(a.Tc, ct0 + fa.S) - ct0;
      const int rot = chunk_rot(cnt);
      for (int k = 0; k < cnt; ++k, ++i) {
        const int ct = ct0 + (rot + k) % cnt;
        const int buf = static_cast<int>(i & 1);
        const uint32_t tph = static_cast<uint32_t>((i >> 1) & 1);
        const bool got = mbar_wait(&tfull[buf], tph, abort_flag);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int col0 = ct * BN;
        const int nvalid = min(BN, a.K - col0);
#pragma unroll 1
        for (int ch = 0; ch < C::CHUNKS; ++ch) {
          const int ct0 = grp * C::COLS + ch * 32;
          uint32_t vv[32];
          tmem_ld_32x32(lane_base + static_cast<uint32_t>(buf * BN + ct0), vv);
          tmem_ld_wait();
          if (ch == C::CHUNKS - 1) {
            tc_fence_before();
            if constexpr (PAIR)
              mbar_arrive_cluster(tempty_l + buf * 8);
            else
              mbar_arrive(&tempty[buf]);
          }
          const int c0 = col0 + ct0;
          float d[32];
          if (ct0 + 32 <= nvalid) {
#pragma unroll
            for (int q = 0; q < 32; ++q) d[q] = __uint_as_float(vv[q]);
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) d[q] = (ct0 + q < nvalid) ? __uint_as_float(vv[q]) : kPastK;
          }
          float m11[11];
#pragma unroll
          for (int q = 0; q < 10; ++q) m11[q] = fmin3(d[3 * q], d[3 * q + 1], d[3 * q + 2]);
          m11[10] = fminf(d[30], d[31]);
          const float m4a = fmin3(m11[0], m11[1], m11[2]), m4b = fmin3(m11[3], m11[4], m11[5]);
          const float m4c = fmin3(m11[6], m11[7], m11[8]), m4d = fminf(m11[9], m11[10]);
          const float m = fminf(fmin3(m4a, m4b, m4c), m4d);
          const unsigned need = __ballot_sync(0xffffffffu, m < bd[TOPK - 1]);
          if (__popc(need) >= kMergeLanes) {
            topk_merge_chunk(bd, bi, d, c0);
          } else if (need) {
            topk_insert_few(bd, bi, d, c0);
          }
        }
      }
      if (!ok) break;
      // ---- flush: merge the column groups, write slot j of row tile rt
      if constexpr (C::GROUPS > 1) {
        float2 *mine = mbuf + (static_cast<int64_t>(grp - 1) * BM + row_in_tile) * TOPK;
        if (grp > 0) {
          if (nflush > 0 && !mbar_wait(mdone, (nflush - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int q = 0; q < TOPK; ++q) mine[q] = make_float2(bd[q], __int_as_float(bi[q]));
          mbar_arrive(mready);
        } else {
          if (!mbar_wait(mready, nflush & 1u, abort_flag)) {
            ok = false;
            break;
          }
          #pragma unroll 1
          for (int e8 = 0; e8 < (C::GROUPS - 1) * TOPK; ++e8) {
            const float2 e = mbuf[(static_cast<int64_t>(e8 / TOPK) * BM + row_in_tile) * TOPK + e8 % TOPK];
            if (e.x < bd[TOPK - 1]) topk_insert(bd, bi, e.x, __float_as_int(e.y));
          }
          mbar_arrive(mdone);
        }
      }
      ++nflush;
      if (grp == 0 && rows_here) {
        // the slot is rewritten only after every certificate task of (l-1, rt) has read it
        bool got = true;
        if (lane == 0 && settled_prev < tile_rows(rt))
          got = wait_count(fa.cert_done + (l - 1) * RT + rt, tile_rows(rt), progress, abort_flag);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        const int64_t n = rt * BM + row_in_tile;
        if (n < a.N) {
          float4 *out = reinterpret_cast<float4 *>(a.cand + ((rt * a.maxs + j) * BM + row_in_tile) * TOPK);
#pragma unroll
          for (int q = 0; q < TOPK; ++q)
            if (bi[q] >= a.K) {
              bd[q] = inf_f();
              bi[q] = -1;
            }
#pragma unroll
          for (int q = 0; q < TOPK; q += 2)
            out[q / 2] = make_float4(2.f * bd[q], __int_as_float(bi[q]), 2.f * bd[q + 1], __int_as_float(bi[q + 1]));
        }
        warp_release_add<false>(fa.chunk_done + static_cast<int64_t>(l) * RT + rt, 1u, lane);
        if (warp == 0 && lane == 0) atomicAdd(progress, 1u);  // liveness for the bounded waits
      }
    }
    if (!ok) {
      *abort_flag = 1;
      set_status(a.status, RVQ_ERR_TIMEOUT);
    }
  } else if (warp >= CERT0 && !((SKIP >> (warp - CERT0)) & 1)) {
    // ------------------------------------------------------------ certificate warps
    const int64_t cw = static_cast<int64_t>(G) * CW;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * CW + (warp - CERT0) -
                       __popc(SKIP & ((1u << (warp - CERT0)) - 1u));
    const int TG = BM / fa.RPT;
    const int64_t total_tasks = static_cast<int64_t>(fa.L) * RT * TG;
    const uint32_t all_rows = static_cast<uint32_t>(a.N) * static_cast<uint32_t>(fa.L);
    RowArgs ra = r0;  // r0.nslots = NC: a row tile's candidate lists are its chunks' slots
    bool ok = true;

    // Claim and run one slice of a queued row's exact scan; false when none is ready.
    auto help_exact = [&]() -> bool {
      int64_t claimed = -1;
      int en = 0, el = 0;
      if (lane == 0) {
        // plain (relaxed) polling reads; the entry's ready flag is acquired before it is used
        const uint32_t rows = min(*reinterpret_cast<const volatile uint32_t *>(ex_rows),
                                  static_cast<uint32_t>(EXACT_QCAP));
        const uint32_t s = rows ? *reinterpret_cast<const volatile uint32_t *>(ex_next) : 0u;
        if (s < rows * static_cast<uint32_t>(fa.NS)) {
          const int q = static_cast<int>(s / fa.NS);
          if (ld_acquire_gpu(reinterpret_cast<const uint32_t *>(&fa.ex_entry[q].z)) != 0 &&
              atomicCAS(ex_next, s, s + 1) == s) {
            claimed = s;
            const int4 e = __ldcg(fa.ex_entry + q);
            en = e.x;
            el = e.y;
          }
        }
      }
      claimed = __shfl_sync(0xffffffffu, claimed, 0);
      if (claimed < 0) return false;
      const int q = static_cast<int>(claimed / fa.NS), sl = static_cast<int>(claimed % fa.NS);
      const int64_t n = __shfl_sync(0xffffffffu, en, 0);
      const int l = __shfl_sync(0xffffffffu, el, 0);
      RowArgs xa = r0;
      xa.l = l;
      xa.last = l == fa.L - 1;
      xa.src = l == 0 ? r0.src : static_cast<const void *>(r0.R);
      float4 rv[NCH];
#pragma unroll
      for (int k = 0; k < NCH; ++k) {
        const int i = lane * 4 + k * 128;
        rv[k] = i >= a.D ? make_float4(0.f, 0.f, 0.f, 0.f)
                : l == 0 ? ld_src4<SRC0>(xa.src, n * a.D + i) : ld_src4<SRC_R>(xa.src, n * a.D + i);
      }
      const int k0 = sl * fa.slice, k1 = min(a.K, k0 + fa.slice);
      double best;
      int bid;
      exact_slice<CB_BF16, NCH>(xa, n, k0, k1, rv, lane, best, bid);
      uint32_t old = 0;
      if (lane == 0) {
        fa.ex_part[static_cast<int64_t>(q) * fa.NS + sl] = make_double2(best, static_cast<double>(bid));
        __threadfence();
        old = atomicAdd(reinterpret_cast<uint32_t *>(&fa.ex_entry[q].w), 1u);
        __threadfence();
        atomicAdd(progress, 1u);
      }
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old + 1 == static_cast<uint32_t>(fa.NS)) {
        // last slice: reduce (lowest distance, then lowest index) and settle the row
        double b = inf_d();
        int id = 0x7fffffff;
        for (int s2 = lane; s2 < fa.NS; s2 += 32) {
          const double2 pr = __ldcg(fa.ex_part + static_cast<int64_t>(q) * fa.NS + s2);
          const int pid = static_cast<int>(pr.y);
          if (pr.x < b || (pr.x == b && pid < id)) {
            b = pr.x;
            id = pid;
          }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
          const double ob = __shfl_xor_sync(0xffffffffu, b, off);
          const int oi = __shfl_xor_sync(0xffffffffu, id, off);
          if (ob < b || (ob == b && oi < id)) {
            b = ob;
            id = oi;
          }
        }
        if (id < 0 || id >= a.K) {  // only reachable with non-finite inputs
          if (lane == 0) {
            r0.ids[n * r0.L + l] = -1;
            set_status(a.status, RVQ_ERR_ARG);
          }
        } else {
          float4 c[NCH];
          const int64_t coff = (static_cast<int64_t>(l) * a.K + id) * a.D;
#pragma unroll
          for (int k = 0; k < NCH; ++k) {
            const int i = lane * 4 + k * 128;
            c[k] = i < a.D ? ld4<CB_BF16>(r0.cb, coff + i) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          apply_row<NCH>(xa, n, rv, c, id, lane);
        }
        warp_release_add<true>(fa.cert_done + static_cast<int64_t>(l) * RT + n / BM, 1u, lane);
        if (lane == 0) atomicAdd(settled, 1u);
      }
      return true;
    };
    // Wait for *ctr >= target, running exact-scan slices meanwhile.  Each poll reads the
    // (per row tile) counter and, unless the exact-scan queue is empty, its head; the progress
    // word for the time limit is read every 16th poll.
    auto wait_helping = [&](const uint32_t *ctr, uint32_t target) -> bool {
      uint32_t last_p = 0;
      uint64_t t0 = 0;
      bool first = true;
      for (uint32_t iter = 0;; ++iter) {
        uint32_t c = 0;
        if (lane == 0) c = ld_acquire_gpu(ctr);
        c = __shfl_sync(0xffffffffu, c, 0);
        if (c >= target) return true;
        if (*abort_flag) return false;
        if (help_exact()) {
          first = true;
          continue;
        }
        if (first || (iter & 15) == 0) {
          uint32_t pr = 0;
          if (lane == 0) pr = *reinterpret_cast<const volatile uint32_t *>(progress);
          pr = __shfl_sync(0xffffffffu, pr, 0);
          const uint64_t now = global_timer_ns();
          if (first || pr != last_p) {
            first = false;
            last_p = pr;
            t0 = now;
          } else if (now - t0 > 2000000000ull) {
            *abort_flag = 1;
            return false;
          }
        }
        __nanosleep(500);
      }
    };

    for (int64_t s = gw; s < total_tasks && ok; s += cw) {
      const int g = static_cast<int>(s % TG);
      const int64_t rt = (s / TG) % RT;
      const int l = static_cast<int>(s / (TG * RT));
      if (!wait_helping(fa.chunk_done + static_cast<int64_t>(l) * RT + rt, 4u * fa.NC) ||
          (l > 0 && !wait_helping(fa.cert_done + static_cast<int64_t>(l - 1) * RT + rt, tile_rows(rt)))) {
        ok = false;
        break;
      }
      ra.l = l;
      ra.last = l == fa.L - 1;
      ra.stats = fa.level_stats + static_cast<int64_t>(l) * RVQ_LEVEL_STATS;
      ra.src = l == 0 ? r0.src : static_cast<const void *>(r0.R);
      if (l == 0 && rt == 0 && g == 0 && r0.offsets) check_offsets(ra, lane, 32);
      const int64_t n0 = rt * BM + static_cast<int64_t>(g) * fa.RPT;
      const int64_t n1 = min(a.N, n0 + fa.RPT);
      uint32_t done_rows = 0;
      for (int64_t n = n0; n < n1; ++n) {
        const bool settled_row = l == 0 ? rescore_row<CB_BF16, SRC0, NCH>(ra, n, lane)
                                        : rescore_row<CB_BF16, SRC_R, NCH>(ra, n, lane);
        if (settled_row) {
          ++done_rows;
          continue;
        }
        // queue the row's exact scan (or, with the queue full, scan it here)
        uint32_t q = 0;
        if (lane == 0) {
          q = atomicAdd(ex_rows, 1u);
          atomicAdd(fa.fb_level + l, 1);
          if (q < EXACT_QCAP) {
            fa.ex_entry[q] = make_int4(static_cast<int>(n), l, 0, 0);
            __threadfence();
            atomicExch(reinterpret_cast<uint32_t *>(&fa.ex_entry[q].z), 1u);
          }
        }
        q = __shfl_sync(0xffffffffu, q, 0);
        if (q >= EXACT_QCAP) {
          if (l == 0)
            exact_row<CB_BF16, SRC0, NCH>(ra, n, lane);
          else
            exact_row<CB_BF16, SRC_R, NCH>(ra, n, lane);
          ++done_rows;
        }
      }
      warp_release_add<true>(fa.cert_done + static_cast<int64_t>(l) * RT + rt, done_rows, lane);
      if (lane == 0) {
        if (done_rows) atomicAdd(settled, done_rows);
        atomicAdd(progress, 1u);
      }
    }
    // help with the remaining exact scans until every row of every level is settled
    if (ok && !wait_helping(settled, all_rows)) ok = false;
    if (!ok) {
      *abort_flag = 1;
      set_status(a.status, RVQ_ERR_TIMEOUT);
    }
  }

  // no bulk copy or MMA may still be in flight when the block exits (a pair's MMAs and bytes are
  // counted on the leader's barriers, so the leader waits for both CTAs)
  if (warp == C::ISSUER && lane == 0 && rank == 0) {
    if constexpr (PAIR)
      umma_commit_pair(mma_done);
    else
      umma_commit(mma_done);
    mbar_wait(mma_done, 0, never);
  }
  if (warp == C::PRODUCER && lane == 0 && *abort_flag && rank == 0) {
    const int64_t pending = p_issued < NSTAGE ? p_issued : NSTAGE;
    for (int64_t jj = 0; jj < pending; ++jj) {
      int back = p_s - 1 - static_cast<int>(jj);
      uint32_t ph = p_ph;
      while (back < 0) {
        back += NSTAGE;
        ph ^= 1u;
      }
      mbar_wait(&full[back], ph, never);
    }
  }
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the peer may signal this CTA's barriers until both are done
  tc_fence_after();
  if (warp == C::ISSUER) {
    __syncwarp();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host plan

struct Plan {
  int64_t RT;  // 128-row tiles
  int Tc;
  int64_t U;
  int G;       // CTAs
  int maxs;    // partial-list slots per row tile (the larger of the two paths' needs)
  // all levels in one launch with every CTA resident (encode_flow_kernel)
  bool flow;
  int L;
  int NC, S;      // chunks per row tile, codeword tiles per chunk
  int RPT;        // rows per certificate task
  int NS, slice;  // exact-scan slices per queued row, codewords per slice
  int Gf;         // CTAs of the flow launch (one per SM)
  bool fpair;     // the flow launch runs CTA pairs (cta_group::2) over 256-row units
};

// Smallest batch that the all-levels kernel runs as CTA pairs.  Pairs halve each SM's codeword
// tile traffic and draw less power, which pays under the power cap of a long launch (2^20 rows
// of D = 1024, L = 8, K = 16384: 222 vs 238 ms; 206181 rows, L = 8: 45 vs 46.5 ms; 16352 rows:
// 3.56-3.65 vs 3.70-3.72 ms); at 4096 rows (L = 4, K = 8192) the two run the same.
constexpr int64_t kPairMinRows = 8192;

inline bool flow_pairs_fit(int grid);

// RVQ_PERSISTENT=0 keeps the per-level launches for every width (tuning / comparison knob).
inline bool persistent_enabled() {
  static int v = [] {
    const char *e = getenv("RVQ_PERSISTENT");
    return e ? atoi(e) : 1;
  }();
  return v != 0;
}

// Row chunks (float4 per lane) of the register-resident row kernels for feature width D <= 1024.
inline int row_chunks(int D) { return D <= 128 ? 1 : D <= 256 ? 2 : D <= 512 ? 4 : 8; }

// Slots a row tile of Tc units needs when U units are split into G ranges: every range but the
// last holds at least f = floor(U/G) units, so Tc consecutive units meet at most 1 + ceil((Tc-1)/f).
inline int64_t slots_needed(int64_t U, int64_t G, int64_t Tc) {
  const int64_t f = std::max<int64_t>(1, U / G);
  return std::min<int64_t>(G, 1 + (Tc - 1 + f - 1) / f);
}

inline Plan make_plan(int64_t N, int K, int D, int L, int sms) {
  Plan p;
  p.RT = (N + BM - 1) / BM;
  p.Tc = (K + BN - 1) / BN;
  p.U = p.RT * p.Tc;
  // every CTA covers at least f = floor(U/G) units, so a row tile (Tc consecutive units) meets
  // at most 1 + ceil((Tc-1)/f) CTAs; keep that within the rescore warp's candidate capacity
  const int64_t slots_cap = MAX_SLOTS;
  const int64_t need_f = std::max<int64_t>(1, (p.Tc - 1 + slots_cap - 2) / (slots_cap - 1));
  int64_t G = std::min<int64_t>(sms, p.U);
  G = std::min<int64_t>(G, std::max<int64_t>(1, p.U / need_f));
  p.G = static_cast<int>(G);
  p.maxs = static_cast<int>(slots_needed(p.U, p.G, p.Tc));

  const int nch = row_chunks(D);
  p.L = L;
  // D in (128, 256] and (512, 1024]: 8 epilogue + 5 certificate warps (other widths run the
  // levels one by one)
  p.flow = D <= 1024 && (nch == 2 || nch == 8) && persistent_enabled() &&
           static_cast<uint64_t>(N) * static_cast<uint64_t>(L) < (uint64_t(1) << 32);
  p.NC = p.S = p.RPT = p.NS = p.slice = p.Gf = 0;
  p.fpair = false;
  if (p.flow) {
    p.Gf = sms;
    // CTA pairs halve the codeword-tile traffic of each SM (each CTA of a pair loads half of a
    // tile); they pay on batches long enough to run under the power cap
    p.fpair = nch == 8 && N >= kPairMinRows && flow_pairs_fit(p.Gf);
    const int64_t units = p.fpair ? (p.RT + 1) / 2 : p.RT;
    const int64_t walkers = p.fpair ? p.Gf / 2 : p.Gf;
    // enough chunks per level to keep every walker busy and finish a row tile soon after it starts
    int nc = static_cast<int>(std::min<int64_t>(MAX_SLOTS, std::max<int64_t>(1, (4 * walkers + units - 1) / units)));
    nc = std::min(nc, p.Tc);
    p.S = (p.Tc + nc - 1) / nc;
    p.NC = (p.Tc + p.S - 1) / p.S;  // no empty chunk
    p.maxs = std::max(p.maxs, p.NC);
    // certificate tasks: about two per certificate warp per level, at most one row tile each
    const int64_t cw = static_cast<int64_t>(p.Gf) * (nch == 8 ? FlowCfg<FLOW_EPI_WIDE, FLOW_RW_WIDE, FLOW_SKIP_WIDE>::CERT_WARPS
                                                              : FlowCfg<FLOW_EPI_NARROW, FLOW_RW_NARROW, FLOW_SKIP_NARROW>::CERT_WARPS);
    int tg = 1;
    while (tg < 64 && static_cast<int64_t>(tg) * p.RT < 2 * cw) tg *= 2;
    p.RPT = BM / tg;
    p.slice = std::max(64, (K + EXACT_NS_MAX - 1) / EXACT_NS_MAX);
    p.NS = (K + p.slice - 1) / p.slice;
  }
  return p;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
  size_t R, Rt, rowstat, cand, fb_list, fb_count, sync, sync_end, ex_part, total;
};

// The row state (fp32 residual, its bf16 operand copy, row statistics) opens every workspace;
// its size depends on N and D only.
inline size_t row_state_bytes(int64_t N, int D) {
  return align256(static_cast<size_t>(N) * D * 4) + align256(static_cast<size_t>(N) * D * 2) +
         align256(static_cast<size_t>(N) * 8);
}

inline Layout make_layout(int64_t N, int D, const Plan &p) {
  Layout w;
  size_t off = 0;
  w.R = off;
  off += align256(static_cast<size_t>(N) * D * 4);
  w.Rt = off;
  off += align256(static_cast<size_t>(N) * D * 2);
  w.rowstat = off;
  off += align256(static_cast<size_t>(N) * 8);
  w.cand = off;  // == row_state_bytes(N, D)
  off += align256(static_cast<size_t>(p.RT) * p.maxs * BM * TOPK * 8);
  w.fb_list = off;
  off += align256(static_cast<size_t>(N) * 4);
  w.fb_count = off;
  off += align256(64 * 4);
  w.sync = off;  // directly after fb_count: one memset clears both
  if (p.flow) {  // progress counters, chunk_done [L, RT], cert_done [L, RT], exact-scan queue entries
    off += 256 + align256(2 * static_cast<size_t>(p.L) * p.RT * 4) + align256(EXACT_QCAP * 16);
  }
  w.sync_end = off;
  w.ex_part = off;
  if (p.flow) off += align256(static_cast<size_t>(EXACT_QCAP) * p.NS * 16);
  w.total = off;
  return w;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 [L, K, D] row-major as a 3-D tensor, box = BK x box_rows x 1, 128B swizzle.
inline bool make_map3(CUtensorMap *m, const void *base, int L, int K, int D, int box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(L)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(K) * D * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [rows, D] row-major, box = BK elements x box_rows rows, 128B swizzle, zero fill outside.
inline bool make_map(CUtensorMap *m, const void *base, int64_t rows, int D, int box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


template <int EPI>
inline bool set_gemm_attr() {
  return cudaFuncSetAttribute(dist_topk_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              GemmCfg<EPI>::SMEM) == cudaSuccess;
}

// Epilogue warps of the per-level distance GEMM: 4 above D = 512 (a tile's longer MMA hides a
// 4-warp epilogue: 5% faster than 8 at D = 1024), else 8 (8 beat 16 at D = 256: 31.4 vs 35.0 ms
// per offline level, and 4: 33.2 ms).
inline int epilogue_warps(int D) { return D > 512 ? 4 : 8; }

inline bool gemm_attrs_ready(int epi) {
  static std::once_flag once;
  static bool ok = false;
  std::call_once(once, [] {
    ok = set_gemm_attr<4>() && set_gemm_attr<8>();
  });
  (void)epi;
  return ok;
}

template <int EPI>
inline cudaError_t launch_gemm_t(int groups, cudaStream_t s, const CUtensorMap &tmA, const CUtensorMap &tmB,
                                 const GemmArgs &ga) {
  using C = GemmCfg<EPI>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(groups);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dist_topk_kernel<EPI>, tmA, tmB, ga);
}

// All-levels dataflow encode, instantiated for 2 (D in (128, 256]) and 8 (D in (512, 1024])
// float4 row chunks.

template <int EPI, int RW, int SK, bool CB, bool XB, int NCH, bool PAIR = false>
inline bool set_flow_attr() {
  return cudaFuncSetAttribute(encode_flow_kernel<EPI, RW, SK, CB, XB, NCH, PAIR>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, FlowMem<EPI, PAIR>::SMEM) == cudaSuccess;
}

inline bool flow_attrs_ready() {
  static std::once_flag once;
  static bool ok = false;
  std::call_once(once, [] {
    constexpr int EW = FLOW_EPI_WIDE, RWD = FLOW_RW_WIDE, SW = FLOW_SKIP_WIDE;
    constexpr int EN = FLOW_EPI_NARROW, RN = FLOW_RW_NARROW, SN = FLOW_SKIP_NARROW;
    ok = set_flow_attr<EW, RWD, SW, false, false, 8>() && set_flow_attr<EW, RWD, SW, false, true, 8>() &&
         set_flow_attr<EW, RWD, SW, true, false, 8>() && set_flow_attr<EW, RWD, SW, true, true, 8>() &&
         set_flow_attr<EW, RWD, SW, false, false, 8, true>() && set_flow_attr<EW, RWD, SW, false, true, 8, true>() &&
         set_flow_attr<EW, RWD, SW, true, false, 8, true>() && set_flow_attr<EW, RWD, SW, true, true, 8, true>() &&
         set_flow_attr<EN, RN, SN, false, false, 2>() && set_flow_attr<EN, RN, SN, false, true, 2>() &&
         set_flow_attr<EN, RN, SN, true, false, 2>() && set_flow_attr<EN, RN, SN, true, true, 2>();
  });
  return ok;
}

// Single CTAs launch cooperatively (every CTA resident: CTAs wait on one another's counters).
// Pairs launch as clusters of two without the cooperative attribute (the profiler refuses a
// cooperative launch with a cluster shape); the plan picks pairs only when the cluster occupancy
// query puts every cluster on the GPU at once, and a CTA that waits on one that never becomes
// resident still gives up with RVQ_ERR_TIMEOUT once nothing has moved for two seconds.
template <int EPI, int RW, int SK, bool PAIR>
inline void flow_launch_config(cudaLaunchConfig_t *cfg, cudaLaunchAttribute (&attr)[1], int grid, cudaStream_t s) {
  *cfg = {};
  cfg->gridDim = dim3(grid);
  cfg->blockDim = dim3(FlowCfg<EPI, RW, SK>::THREADS);
  cfg->dynamicSmemBytes = FlowMem<EPI, PAIR>::SMEM;
  cfg->stream = s;
  if constexpr (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
  } else {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  }
  cfg->attrs = attr;
  cfg->numAttrs = 1;
}

// Whether `grid` CTAs of the pair kernel for D in (512, 1024] can all be resident as 2-CTA clusters.
inline bool flow_pairs_fit(int grid) {
  static std::once_flag once;
  static int clusters = 0;
  std::call_once(once, [] {
    if (!flow_attrs_ready()) return;
    constexpr int EW = FLOW_EPI_WIDE, RWD = FLOW_RW_WIDE, SW = FLOW_SKIP_WIDE;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    flow_launch_config<EW, RWD, SW, true>(&cfg, attr, 2, nullptr);
    if (cudaOccupancyMaxActiveClusters(&clusters, encode_flow_kernel<EW, RWD, SW, true, true, 8, true>, &cfg) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      clusters = 0;
    }
  });
  return grid % 2 == 0 && clusters >= grid / 2;
}

template <int EPI, int RW, int SK, bool CB, bool XB, int NCH, bool PAIR = false>
inline cudaError_t launch_flow_t(int grid, cudaStream_t s, const CUtensorMap &tmA0, const CUtensorMap &tmA,
                                 const CUtensorMap &tmB3, const GemmArgs &ga, const RowArgs &ra, const FlowArgs &fa) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  flow_launch_config<EPI, RW, SK, PAIR>(&cfg, attr, grid, s);
  return cudaLaunchKernelEx(&cfg, encode_flow_kernel<EPI, RW, SK, CB, XB, NCH, PAIR>, tmA0, tmA, tmB3, ga, ra, fa);
}

inline cudaError_t launch_flow(int nch, bool pair, bool cb_bf16, bool x_bf16, int grid, cudaStream_t s,
                               const CUtensorMap &tmA0, const CUtensorMap &tmA, const CUtensorMap &tmB3,
                               const GemmArgs &ga, const RowArgs &ra, const FlowArgs &fa) {
  constexpr int EW = FLOW_EPI_WIDE, RWD = FLOW_RW_WIDE, SW = FLOW_SKIP_WIDE;
  constexpr int EN = FLOW_EPI_NARROW, RN = FLOW_RW_NARROW, SN = FLOW_SKIP_NARROW;
  if (pair) {
    if (nch != 8) return cudaErrorInvalidValue;
    if (cb_bf16) return x_bf16 ? launch_flow_t<EW, RWD, SW, true, true, 8, true>(grid, s, tmA0, tmA, tmB3, ga, ra, fa)
                               : launch_flow_t<EW, RWD, SW, true, false, 8, true>(grid, s, tmA0, tmA, tmB3, ga, ra, fa);
    return x_bf16 ? launch_flow_t<EW, RWD, SW, false, true, 8, true>(grid, s, tmA0, tmA, tmB3, ga, ra, fa)
                  : launch_flow_t<EW, RWD, SW, false, false, 8, true>(grid, s, tmA0, tmA, tmB3, ga, ra, fa);
  }
  if (nch == 2) {
    if (cb_bf16) return x_bf16 ? launch_flow_t<EN, RN, SN, true, true, 2>(grid, s, tmA0, tmA, tmB3, ga, ra, fa)
                               : launch_flow_t<EN, RN, SN, true, false, 2>(grid, s, tmA0, tmA, tmB3, ga, ra, fa);
    return x_bf16 ? launch_flow_t<EN, RN, SN, false, true, 2>(grid, s, tmA0, tmA, tmB3, ga, ra, fa)
                  : launch_flow_t<EN, RN, SN, false, false, 2>(grid, s, tmA0, tmA, tmB3, ga, ra, fa);
  }
  if (nch != 8) return cudaErrorInvalidValue;
  if (cb_bf16) return x_bf16 ? launch_flow_t<EW, RWD, SW, true, true, 8>(grid, s, tmA0, tmA, tmB3, ga, ra, fa)
                             : launch_flow_t<EW, RWD, SW, true, false, 8>(grid, s, tmA0, tmA, tmB3, ga, ra, fa);
  return x_bf16 ? launch_flow_t<EW, RWD, SW, false, true, 8>(grid, s, tmA0, tmA, tmB3, ga, ra, fa)
                : launch_flow_t<EW, RWD, SW, false, false, 8>(grid, s, tmA0, tmA, tmB3, ga, ra, fa);
}

inline cudaError_t launch_gemm(int epi, int groups, cudaStream_t s, const CUtensorMap &tmA, const CUtensorMap &tmB,
                               const GemmArgs &ga) {
  if (epi == 4) return launch_gemm_t<4>(groups, s, tmA, tmB, ga);
  return launch_gemm_t<8>(groups, s, tmA, tmB, ga);
}

}  // namespace enc
}  // namespace rvq

extern "C" int rvq_encode_workspace_size(int64_t N, int D, int L, int K, size_t *bytes) {
  RVQ_ENTRY("rvq_encode_workspace_size");
  using namespace rvq;
  if (!bytes || N < 0 || D < 1 || L < 1 || K < 1) return RVQ_ERR_ARG;
  if (L > 64 || D < 64 || D > 4096 || D % 64 != 0 || N >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  int sms = 0;
  int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  const enc::Plan p = enc::make_plan(std::max<int64_t>(N, 1), K, D, L, sms);
  *bytes = enc::make_layout(N, D, p).total;
  return RVQ_OK;
}

extern "C" int rvq_encode_levels_per_launch(int64_t N, int D, int L, int K, int *levels) {
  using namespace rvq;
  if (!levels || N < 0 || D < 1 || L < 1 || K < 1) return RVQ_ERR_ARG;
  if (L > 64 || D < 64 || D > 4096 || D % 64 != 0 || N >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  int sms = 0;
  int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  const enc::Plan p = enc::make_plan(std::max<int64_t>(N, 1), K, D, L, sms);
  *levels = p.flow ? L : 1;
  return RVQ_OK;
}

extern "C" int rvq_encode_candidate_layout(int64_t N, int D, int L, int K, size_t *offset, int *slots) {
  using namespace rvq;
  if (!offset || !slots || N < 0 || D < 1 || L < 1 || K < 1) return RVQ_ERR_ARG;
  if (L > 64 || D < 64 || D > 4096 || D % 64 != 0 || N >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  int sms = 0;
  int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  const enc::Plan p = enc::make_plan(std::max<int64_t>(N, 1), K, D, L, sms);
  *offset = enc::make_layout(N, D, p).cand;
  *slots = p.maxs;
  return RVQ_OK;
}

extern "C" int rvq_encode(const void *features, int f_dtype, int64_t N, int D, const void *codebooks, int cb_dtype,
                          const void *cb_operand, const float *norms, const float *level_stats, int L, int K,
                          const int64_t *offsets, int64_t B, int32_t *ids, float *residual, float *recon,
                          int32_t *fallbacks, void *workspace, size_t workspace_bytes, int32_t *status,
                          void *stream) {
  RVQ_ENTRY("rvq_encode");
  using namespace rvq;
  using namespace rvq::enc;
  if (N < 0 || D < 1 || L < 1 || K < 1 || B < 0) return RVQ_ERR_ARG;
  if ((f_dtype != RVQ_F32 && f_dtype != RVQ_BF16) || (cb_dtype != RVQ_F32 && cb_dtype != RVQ_BF16))
    return RVQ_ERR_ARG;
  if (L > 64 || D < 64 || D > 4096 || D % 64 != 0 || N >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  if (offsets == nullptr && B != 0) return RVQ_ERR_ARG;
  if (N == 0) return RVQ_OK;
  if (!features || !codebooks || !norms || !level_stats || !ids) return RVQ_ERR_ARG;
  if (cb_dtype == RVQ_F32 && !cb_operand) return RVQ_ERR_ARG;
  const void *op = cb_dtype == RVQ_BF16 ? codebooks : cb_operand;
  if (!aligned16(features) || !aligned16(codebooks) || !aligned16(op) || !aligned16(norms) ||
      (residual && !aligned16(residual)) || (recon && !aligned16(recon)) || (reinterpret_cast<uintptr_t>(ids) & 3u))
    return RVQ_ERR_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RVQ_ERR_WORKSPACE;
  int sms = 0;
  int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  const Plan p = make_plan(N, K, D, L, sms);
  const Layout w = make_layout(N, D, p);
  if (workspace_bytes < w.total) return RVQ_ERR_WORKSPACE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *R = residual ? residual : reinterpret_cast<float *>(ws + w.R);
  __nv_bfloat16 *Rt = reinterpret_cast<__nv_bfloat16 *>(ws + w.Rt);
  float2 *rowstat = reinterpret_cast<float2 *>(ws + w.rowstat);
  float2 *cand = reinterpret_cast<float2 *>(ws + w.cand);
  int32_t *fb_list = reinterpret_cast<int32_t *>(ws + w.fb_list);
  int32_t *fb_count = reinterpret_cast<int32_t *>(ws + w.fb_count);

  CUtensorMap tmA;
  if (!make_map(&tmA, Rt, N, D, BM)) return RVQ_ERR_CUDA;

  const int epi = epilogue_warps(D);
  if (!gemm_attrs_ready(epi)) return RVQ_ERR_CUDA;

  // D <= 1024: register-resident row kernels; level 0 reads the features directly (bf16 features
  // are their own tensor-core operand, so no initial copy at all).  Wider rows: the init kernel
  // materialises the fp32 residual and the row kernels stream it.
  const bool fast = D <= 1024;
  const int nch = row_chunks(D);
  const bool x_is_operand = fast && f_dtype == RVQ_BF16;
  if (!x_is_operand) {
    const int64_t threads = N * 32;
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    cudaError_t e;
    if (fast)  // only the level-0 operand copy and row statistics
      e = launch_pdl(init_kernel<false, false>, dim3(blocks), dim3(256), 0, s, features, N, D, R, Rt, rowstat,
                     fb_count, 0, static_cast<const int64_t *>(nullptr), int64_t(0), status);
    else if (f_dtype == RVQ_BF16)
      e = launch_pdl(init_kernel<true, true>, dim3(blocks), dim3(256), 0, s, features, N, D, R, Rt, rowstat,
                     fb_count, L, offsets, B, status);
    else
      e = launch_pdl(init_kernel<false, true>, dim3(blocks), dim3(256), 0, s, features, N, D, R, Rt, rowstat,
                     fb_count, L, offsets, B, status);
    note_launch();
    if (e != cudaSuccess) return RVQ_ERR_CUDA;
  }
  CUtensorMap tmX;
  if (x_is_operand && !make_map(&tmX, features, N, D, BM)) return RVQ_ERR_CUDA;

  // D in (128, 256] or (512, 1024]: every level in one launch (CTA pairs for long batches at D > 512).
  const bool all_levels = fast && p.flow;
  if (all_levels) {
    if (!flow_attrs_ready()) return RVQ_ERR_CUDA;
    CUtensorMap tmB3;
    if (!make_map3(&tmB3, op, L, K, D, p.fpair ? BN / 2 : BN)) return RVQ_ERR_CUDA;
    if (cudaMemsetAsync(fb_count, 0, w.sync_end - w.fb_count, s) != cudaSuccess) return RVQ_ERR_CUDA;
    uint8_t *sync = ws + w.sync;
    GemmArgs ga;
    ga.norms = norms;
    ga.N = N;
    ga.K = K;
    ga.D = D;
    ga.U = 0;  // chunks, not unit ranges: FlowArgs
    ga.Tc = p.Tc;
    ga.G = p.Gf;
    ga.maxs = p.maxs;
    ga.cand = cand;
    ga.status = status;
    ga.zero_counter = nullptr;
    RowArgs r0;
    r0.N = N;
    r0.D = D;
    r0.K = K;
    r0.L = L;
    r0.l = 0;
    r0.Tc = p.Tc;
    r0.G = p.Gf;
    r0.maxs = p.maxs;
    r0.U = 0;
    r0.rt0 = 0;
    r0.nslots = p.NC;
    r0.cand = cand;
    r0.rowstat = rowstat;
    r0.R = R;
    r0.Rt = Rt;
    r0.cb = codebooks;
    r0.stats = level_stats;
    r0.ids = ids;
    r0.fb_list = nullptr;  // uncertified rows go to the kernel's exact-scan queue
    r0.fb_count = fb_count;
    r0.status = status;
    r0.last = L == 1;
    r0.src = features;
    r0.fb_next = nullptr;
    r0.offsets = offsets;
    r0.B = B;
    FlowArgs fa;
    fa.L = L;
    fa.RT = p.RT;
    fa.NC = p.NC;
    fa.S = p.S;
    fa.RPT = p.RPT;
    fa.NS = p.NS;
    fa.slice = p.slice;
    fa.ctr = reinterpret_cast<uint32_t *>(sync);
    fa.chunk_done = reinterpret_cast<uint32_t *>(sync + 256);
    fa.cert_done = fa.chunk_done + static_cast<size_t>(L) * p.RT;
    fa.ex_entry = reinterpret_cast<int4 *>(sync + 256 + align256(2 * static_cast<size_t>(L) * p.RT * 4));
    fa.ex_part = reinterpret_cast<double2 *>(ws + w.ex_part);
    fa.fb_level = fb_count;
    fa.norms = norms;
    fa.level_stats = level_stats;
    profile_begin(s);
    const cudaError_t fe = launch_flow(nch, p.fpair, cb_dtype == RVQ_BF16, f_dtype == RVQ_BF16, p.Gf, s,
                                       x_is_operand ? tmX : tmA, tmA, tmB3, ga, r0, fa);
    profile_end(s, L);
    note_launch();
    if (fe != cudaSuccess) return RVQ_ERR_CUDA;
  }

  const int64_t row_blocks = (N * 32 + 255) / 256;
  const int fb_blocks = 2 * sms;
  const size_t fb_smem = static_cast<size_t>(D) * sizeof(double);
  for (int l = 0; l < L && !all_levels; ++l) {
    const size_t lvl = static_cast<size_t>(l) * K * D * 2;
    CUtensorMap tmB;
    if (!make_map(&tmB, static_cast<const uint8_t *>(op) + lvl, K, D, BN)) return RVQ_ERR_CUDA;
    GemmArgs ga;
    ga.norms = norms + static_cast<size_t>(l) * K;
    ga.N = N;
    ga.K = K;
    ga.D = D;
    ga.U = p.U;
    ga.Tc = p.Tc;
    ga.G = p.G;
    ga.maxs = p.maxs;
    ga.cand = cand;
    ga.status = status;
    ga.zero_counter = (fast && l == 0) ? fb_count : nullptr;
    profile_begin(s);
    const cudaError_t ge = launch_gemm(epi, p.G, s, (x_is_operand && l == 0) ? tmX : tmA, tmB, ga);
    profile_end(s);
    note_launch();
    if (ge != cudaSuccess) return RVQ_ERR_CUDA;

    RowArgs ra;
    ra.N = N;
    ra.D = D;
    ra.K = K;
    ra.L = L;
    ra.l = l;
    ra.Tc = p.Tc;
    ra.G = p.G;
    ra.maxs = p.maxs;
    ra.U = p.U;
    ra.rt0 = 0;
    ra.nslots = 0;
    ra.cand = cand;
    ra.rowstat = rowstat;
    ra.R = R;
    ra.Rt = Rt;
    ra.cb = codebooks;
    ra.stats = level_stats + static_cast<size_t>(l) * RVQ_LEVEL_STATS;
    ra.ids = ids;
    ra.fb_list = fb_list;
    ra.fb_count = fb_count + l;
    ra.status = status;
    ra.last = l == L - 1;
    ra.src = l == 0 && fast ? features : static_cast<const void *>(R);
    ra.fb_next = (fast && l + 1 < L) ? fb_count + l + 1 : nullptr;
    ra.offsets = (fast && l == 0) ? offsets : nullptr;
    ra.B = B;
    cudaError_t e1 = cudaSuccess, e2 = cudaSuccess;
    if (fast) {
      const unsigned rb = static_cast<unsigned>(row_blocks);
      if (l > 0)
        e1 = cb_dtype == RVQ_BF16 ? launch_rows_fast<true, SRC_R>(ra, nch, rb, fb_blocks, fb_smem, s)
                                  : launch_rows_fast<false, SRC_R>(ra, nch, rb, fb_blocks, fb_smem, s);
      else if (f_dtype == RVQ_BF16)
        e1 = cb_dtype == RVQ_BF16 ? launch_rows_fast<true, SRC_X_BF16>(ra, nch, rb, fb_blocks, fb_smem, s)
                                  : launch_rows_fast<false, SRC_X_BF16>(ra, nch, rb, fb_blocks, fb_smem, s);
      else
        e1 = cb_dtype == RVQ_BF16 ? launch_rows_fast<true, SRC_X_F32>(ra, nch, rb, fb_blocks, fb_smem, s)
                                  : launch_rows_fast<false, SRC_X_F32>(ra, nch, rb, fb_blocks, fb_smem, s);
    } else if (cb_dtype == RVQ_BF16) {
      e1 = launch_pdl(rescore_kernel<true>, dim3(static_cast<unsigned>(row_blocks)), dim3(256), 0, s, ra);
      e2 = launch_pdl(fallback_kernel<true>, dim3(fb_blocks), dim3(256), fb_smem, s, ra);
    } else {
      e1 = launch_pdl(rescore_kernel<false>, dim3(static_cast<unsigned>(row_blocks)), dim3(256), 0, s, ra);
      e2 = launch_pdl(fallback_kernel<false>, dim3(fb_blocks), dim3(256), fb_smem, s, ra);
    }
    note_launch(2);
    if (e1 != cudaSuccess || e2 != cudaSuccess) return RVQ_ERR_CUDA;
  }
  if (fallbacks) {
    if (cudaMemcpyAsync(fallbacks, fb_count, sizeof(int32_t) * L, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return RVQ_ERR_CUDA;
  }
  if (recon) {
    st = launch_decode(ids, N, L, codebooks, cb_dtype, K, D, recon, status, s);
    if (st != RVQ_OK) return st;
  }
  return RVQ_OK;
}

// ---------------------------------------------------------------- encode without a caller workspace
namespace rvq {
namespace enc {

// Scratch of rvq_encode_noalloc: one statically sized array per device, shared by all calls.
static __device__ __align__(256) uint8_t g_noalloc_scratch[RVQ_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device (host code cannot use the symbol
// itself).  It is looked up with that device current the first time the device is used, and again
// whenever the device's current context is a different one (cudaDeviceReset destroys the primary
// context, and the module, with the array in it, is loaded anew at another address).  Contexts are
// told apart by their process-unique id (cuCtxGetId), so a handle value reused by a later context
// cannot bring back a stale address.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

inline bool current_context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

inline int noalloc_scratch(void **ptr) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RVQ_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);  // false before the runtime made a context current
  if (!addr[dev] || !have_ctx || ctx != ctx_of[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RVQ_ERR_CUDA;
    if (!current_context_id(&ctx)) return RVQ_ERR_CUDA;  // the lookup made the primary context current
    addr[dev] = p;
    ctx_of[dev] = ctx;
  }
  *ptr = addr[dev];
  return RVQ_OK;
}

}  // namespace enc
}  // namespace rvq

extern "C" int rvq_encode_noalloc(const void *features, int f_dtype, int64_t N, int D, const void *codebooks,
                                  int cb_dtype, const void *cb_operand, const float *norms, const float *level_stats,
                                  int L, int K, const int64_t *offsets, int64_t B, int32_t *ids, float *residual,
                                  float *recon, int32_t *fallbacks, int32_t *status, void *stream) {
  RVQ_ENTRY("rvq_encode_noalloc");
  size_t need = 0;
  int st = rvq_encode_workspace_size(N, D, L, K, &need);
  if (st != RVQ_OK) return st;
  if (need > RVQ_NOALLOC_SCRATCH_BYTES) return RVQ_ERR_WORKSPACE;
  void *scratch = nullptr;
  st = rvq::enc::noalloc_scratch(&scratch);
  if (st != RVQ_OK) return st;
  return rvq_encode(features, f_dtype, N, D, codebooks, cb_dtype, cb_operand, norms, level_stats, L, K, offsets, B,
                    ids, residual, recon, fallbacks, scratch, RVQ_NOALLOC_SCRATCH_BYTES, status, stream);
}

// ---------------------------------------------------------------- codebook-sharded encode
//
// The codebook axis split over W ranks: rank w holds codewords [k0_w, k0_w + K_w) of every level
// (k0_w = K_0 + ... + K_{w-1}) and all N rows.  Per level:
//   select (each rank): the distance GEMM over the shard, then shard_select_kernel certifies each
//     row's candidates and rescans them exactly, writing the shard's nearest codeword with its
//     exact distance ||r - c||^2; rows the certificate cannot settle get an exact scan of the
//     shard (shard_fallback_kernel).
//   exchange (caller): every rank gathers the W per-rank arrays.
//   apply (each rank): shard_apply_kernel takes the lowest (distance, id) pair of each row, reads
//     that codeword from its owner's shard (a peer pointer when the owner is another GPU) and
//     updates the replicated residual exactly like the single-GPU path, so the replicas stay
//     bit-identical.
// The nearest codeword over all K is the nearest among the shards' nearest ones (ties to the
// lowest id, which is also the lowest rank), so the ids are those of the one-GPU encode.
namespace rvq {
namespace enc {

// One lane's share of ||r - c||^2 with every rounding explicit (no contraction), so that all
// callers get bit-identical distances for equal rows: equal codewords held by different shards
// tie exactly and go to the lowest id.
template <int NCH>
__device__ __forceinline__ double lane_sq_dist(const float4 (&rv)[NCH], const float4 (&c)[NCH]) {
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const double e0 = static_cast<double>(rv[k].x) - c[k].x, e1 = static_cast<double>(rv[k].y) - c[k].y;
    const double e2 = static_cast<double>(rv[k].z) - c[k].z, e3 = static_cast<double>(rv[k].w) - c[k].w;
    const double q = __dadd_rn(__dadd_rn(__dadd_rn(__dmul_rn(e0, e0), __dmul_rn(e1, e1)), __dmul_rn(e2, e2)),
                               __dmul_rn(e3, e3));
    s = __dadd_rn(s, q);
  }
  return s;
}

template <int SRC, int NCH>
__device__ __forceinline__ void load_row(const RowArgs &a, int64_t n, float4 (&rv)[NCH], int lane) {
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int i = lane * 4 + k * 128;
    rv[k] = i < a.D ? ld_src4<SRC>(a.src, n * a.D + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <bool CB_BF16, int NCH>
__device__ __forceinline__ void load_codeword(const void *cb, int64_t coff, int D, float4 (&c)[NCH], int lane) {
#pragma unroll
  for (int k = 0; k < NCH; ++k) {
    const int i = lane * 4 + k * 128;
    c[k] = i < D ? ld4<CB_BF16>(cb, coff + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Nearest codeword of this shard for row n and its exact distance (one warp), from the shard's
// candidate lists: same certificate as rescore_row, but the winner is always rescored exactly
// because its distance is compared with the other shards'.  Uncertified rows are queued.
template <bool CB_BF16, int SRC, int NCH>
__device__ __forceinline__ void shard_best_row(const RowArgs &a, int64_t k0, double2 *sel, int64_t n, int lane) {
  const int64_t rt = n / BM;
  const int rin = static_cast<int>(n - rt * BM);
  const int64_t ut = rt - a.rt0;
  const int c0 = cta_of_unit(ut * a.Tc, a.U, a.G);
  const int c1 = cta_of_unit(ut * a.Tc + a.Tc - 1, a.U, a.G);
  const int ncand = (c1 - c0 + 1) * TOPK;

  float4 rv[NCH];
  load_row<SRC, NCH>(a, n, rv, lane);
  float dv[CPL];
  int iv[CPL];
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    const int e = lane + 32 * h;
    dv[h] = inf_f();
    iv[h] = -1;
    if (e < ncand) {
      const int slot = e / TOPK, t = e - slot * TOPK;
      const float2 c = __ldcg(a.cand + ((rt * a.maxs + slot) * BM + rin) * TOPK + t);
      dv[h] = c.x;
      iv[h] = __float_as_int(c.y);
    }
  }
  float2 rs = make_float2(0.f, 0.f);
  if constexpr (SRC == SRC_X_BF16) {
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < NCH; ++k) q += rv[k].x * rv[k].x + rv[k].y * rv[k].y + rv[k].z * rv[k].z + rv[k].w * rv[k].w;
    rs = make_float2(0.f, __fsqrt_ru(1.0001f * warp_sum_f(q)));
  } else {
    rs = __ldcg(a.rowstat + n);
  }

  float tl = inf_f(), ml = inf_f();
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    const int e = lane + 32 * h;
    if (e < ncand && (e % TOPK) == TOPK - 1) tl = fminf(tl, dv[h]);
    ml = fminf(ml, dv[h]);
  }
  const float T = warp_min_f(tl);
  const float dmin = warp_min_f(ml);
  const float E = error_bound(a.stats, rs, a.D) + 7.62939453125e-06f * (fabsf(dmin) + (T < 1e30f ? fabsf(T) : 0.f));
  const float lim = dmin + 2.f * E;

  double rr = 0.0;
#pragma unroll
  for (int k = 0; k < NCH; ++k)
    rr += static_cast<double>(rv[k].x) * rv[k].x + static_cast<double>(rv[k].y) * rv[k].y +
          static_cast<double>(rv[k].z) * rv[k].z + static_cast<double>(rv[k].w) * rv[k].w;
  rr = warp_sum_d(rr);
  double best = inf_d();
  int best_id = 0x7fffffff;
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    unsigned mask = __ballot_sync(0xffffffffu, iv[h] >= 0 && dv[h] <= lim);
    while (mask) {
      const int srcl = __ffs(mask) - 1;
      mask &= mask - 1;
      const int id = __shfl_sync(0xffffffffu, iv[h], srcl);
      float4 c[NCH];
      load_codeword<CB_BF16, NCH>(a.cb, (static_cast<int64_t>(a.l) * a.K + id) * a.D, a.D, c, lane);
      const double dd = warp_sum_d(lane_sq_dist<NCH>(rv, c));
      if (dd < best || (dd == best && id < best_id)) {
        best = dd;
        best_id = id;
      }
    }
  }
  const bool certified = best_id != 0x7fffffff && (best - rr) < (static_cast<double>(T) - static_cast<double>(E));
  if (!certified) {
    if (lane == 0) {
      const int pos = atomicAdd(a.fb_count, 1);
      a.fb_list[pos] = static_cast<int32_t>(n);
    }
    return;
  }
  if (lane == 0) sel[n] = make_double2(best, static_cast<double>(k0 + best_id));
}

template <bool CB_BF16, int SRC, int NCH>
__global__ void __launch_bounds__(256, 2) shard_select_kernel(const RowArgs a, int64_t k0, double2 *sel) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t n = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (n >= a.N) return;
  shard_best_row<CB_BF16, SRC, NCH>(a, k0, sel, n, threadIdx.x & 31);
}

// Exact scan of the shard's K codewords for each queued row (the block's 8 warps split the
// codewords; every warp keeps the row in registers).  Writes (distance, global id), or (+inf, -1)
// when no distance compares (non-finite inputs).
template <bool CB_BF16, int SRC, int NCH>
__global__ void __launch_bounds__(256) shard_fallback_kernel(const RowArgs a, int64_t k0, double2 *sel) {
  constexpr int NW = 8;
  __shared__ double wbest[NW];
  __shared__ int wid[NW];
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int count = *a.fb_count;
  for (int j = blockIdx.x; j < count; j += gridDim.x) {
    const int64_t n = a.fb_list[j];
    float4 rv[NCH];
    load_row<SRC, NCH>(a, n, rv, lane);
    double bd = inf_d();
    int bk = 0x7fffffff;
    for (int k = warp; k < a.K; k += NW) {
      float4 c[NCH];
      load_codeword<CB_BF16, NCH>(a.cb, (static_cast<int64_t>(a.l) * a.K + k) * a.D, a.D, c, lane);
      const double d = warp_sum_d(lane_sq_dist<NCH>(rv, c));
      if (d < bd) {  // k ascends within a warp: the first of equal distances stays
        bd = d;
        bk = k;
      }
    }
    if (lane == 0) {
      wbest[warp] = bd;
      wid[warp] = bk;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double b = wbest[0];
      int k = wid[0];
      for (int w = 1; w < NW; ++w)
        if (wbest[w] < b || (wbest[w] == b && wid[w] < k)) {
          b = wbest[w];
          k = wid[w];
        }
      sel[n] = k == 0x7fffffff ? make_double2(inf_d(), -1.0) : make_double2(b, static_cast<double>(k0 + k));
    }
    __syncthreads();  // wbest is rewritten by the next row
  }
}

struct ShardApplyArgs {
  const double2 *sel;  // [W, N]: each rank's (exact distance, global id) per row
  int W;
  const void *cb[RVQ_MAX_SHARDS];  // rank w's stored codebooks [L, Kw[w], D] (peer pointers allowed)
  int Kw[RVQ_MAX_SHARDS];
  int64_t k0[RVQ_MAX_SHARDS];
};

// Overall nearest codeword of row n (lowest distance, then lowest id) and the residual update.
template <bool CB_BF16, int SRC, int NCH>
__global__ void __launch_bounds__(256, 2) shard_apply_kernel(const RowArgs a, const ShardApplyArgs s) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t n = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (n >= a.N) return;
  double b = inf_d();
  int id = 0x7fffffff, w = -1;
  if (lane < s.W) {
    const double2 v = __ldcg(s.sel + static_cast<int64_t>(lane) * a.N + n);
    const double lo = static_cast<double>(s.k0[lane]);
    if (v.x == v.x && v.y >= lo && v.y < lo + static_cast<double>(s.Kw[lane])) {
      b = v.x;
      id = static_cast<int>(v.y);
      w = lane;
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, b, off);
    const int oi = __shfl_xor_sync(0xffffffffu, id, off);
    const int ow = __shfl_xor_sync(0xffffffffu, w, off);
    if (ow >= 0 && (w < 0 || ob < b || (ob == b && oi < id))) {
      b = ob;
      id = oi;
      w = ow;
    }
  }
  if (w < 0) {  // no rank produced a usable pair: only reachable with non-finite inputs
    if (lane == 0) {
      a.ids[n * a.L + a.l] = -1;
      set_status(a.status, RVQ_ERR_ARG);
    }
    return;
  }
  float4 rv[NCH], c[NCH];
  load_row<SRC, NCH>(a, n, rv, lane);
  load_codeword<CB_BF16, NCH>(s.cb[w], (static_cast<int64_t>(a.l) * s.Kw[w] + (id - s.k0[w])) * a.D, a.D, c, lane);
  apply_row<NCH>(a, n, rv, c, id, lane);
}

inline Plan make_shard_plan(int64_t N, int Ks, int D, int sms) {
  Plan p = make_plan(N, Ks, D, 1, sms);
  p.flow = false;  // one level per call: the per-level distance kernel
  return p;
}

template <bool CB_BF16, int SRC>
inline cudaError_t launch_shard_select(const RowArgs &ra, int64_t k0, double2 *sel, int nch, unsigned row_blocks,
                                       unsigned fb_blocks, cudaStream_t s) {
  cudaError_t e;
  switch (nch) {
    case 1:
      e = launch_pdl(shard_select_kernel<CB_BF16, SRC, 1>, dim3(row_blocks), dim3(256), 0, s, ra, k0, sel);
      if (e == cudaSuccess)
        e = launch_pdl(shard_fallback_kernel<CB_BF16, SRC, 1>, dim3(fb_blocks), dim3(256), 0, s, ra, k0, sel);
      return e;
    case 2:
      e = launch_pdl(shard_select_kernel<CB_BF16, SRC, 2>, dim3(row_blocks), dim3(256), 0, s, ra, k0, sel);
      if (e == cudaSuccess)
        e = launch_pdl(shard_fallback_kernel<CB_BF16, SRC, 2>, dim3(fb_blocks), dim3(256), 0, s, ra, k0, sel);
      return e;
    case 4:
      e = launch_pdl(shard_select_kernel<CB_BF16, SRC, 4>, dim3(row_blocks), dim3(256), 0, s, ra, k0, sel);
      if (e == cudaSuccess)
        e = launch_pdl(shard_fallback_kernel<CB_BF16, SRC, 4>, dim3(fb_blocks), dim3(256), 0, s, ra, k0, sel);
      return e;
    default:
      e = launch_pdl(shard_select_kernel<CB_BF16, SRC, 8>, dim3(row_blocks), dim3(256), 0, s, ra, k0, sel);
      if (e == cudaSuccess)
        e = launch_pdl(shard_fallback_kernel<CB_BF16, SRC, 8>, dim3(fb_blocks), dim3(256), 0, s, ra, k0, sel);
      return e;
  }
}

template <bool CB_BF16, int SRC>
inline cudaError_t launch_shard_apply(const RowArgs &ra, const ShardApplyArgs &sa, int nch, unsigned row_blocks,
                                      cudaStream_t s) {
  switch (nch) {
    case 1: return launch_pdl(shard_apply_kernel<CB_BF16, SRC, 1>, dim3(row_blocks), dim3(256), 0, s, ra, sa);
    case 2: return launch_pdl(shard_apply_kernel<CB_BF16, SRC, 2>, dim3(row_blocks), dim3(256), 0, s, ra, sa);
    case 4: return launch_pdl(shard_apply_kernel<CB_BF16, SRC, 4>, dim3(row_blocks), dim3(256), 0, s, ra, sa);
    default: return launch_pdl(shard_apply_kernel<CB_BF16, SRC, 8>, dim3(row_blocks), dim3(256), 0, s, ra, sa);
  }
}

// Feature widths of the sharded path: the register-resident row kernels.
inline bool shard_width_ok(int D) { return D >= 64 && D <= 1024 && D % 64 == 0; }

}  // namespace enc
}  // namespace rvq

extern "C" int rvq_shard_workspace_size(int64_t N, int D, int K_shard, size_t *bytes) {
  RVQ_ENTRY("rvq_shard_workspace_size");
  using namespace rvq;
  if (!bytes || N < 0 || D < 1 || K_shard < 1) return RVQ_ERR_ARG;
  if (!enc::shard_width_ok(D) || N >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  int sms = 0;
  const int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  const enc::Plan p = enc::make_shard_plan(std::max<int64_t>(N, 1), K_shard, D, sms);
  *bytes = enc::make_layout(N, D, p).total;
  return RVQ_OK;
}

extern "C" int rvq_shard_select(const void *features, int f_dtype, int64_t N, int D, const void *shard_codebooks,
                                int cb_dtype, const void *shard_operand, const float *shard_norms,
                                const float *shard_stats, int L, int K_shard, int64_t k0, int l, float *residual,
                                double *sel, int32_t *fallbacks, void *workspace, size_t workspace_bytes,
                                int32_t *status, void *stream) {
  RVQ_ENTRY("rvq_shard_select");
  using namespace rvq;
  using namespace rvq::enc;
  if (N < 0 || D < 1 || L < 1 || K_shard < 1 || k0 < 0 || l < 0 || l >= L) return RVQ_ERR_ARG;
  if ((f_dtype != RVQ_F32 && f_dtype != RVQ_BF16) || (cb_dtype != RVQ_F32 && cb_dtype != RVQ_BF16))
    return RVQ_ERR_ARG;
  if (!shard_width_ok(D) || L > 64 || N >= (int64_t(1) << 31) || k0 + K_shard >= (int64_t(1) << 31))
    return RVQ_ERR_UNSUPPORTED;
  if (N == 0) return RVQ_OK;
  if (!features || !shard_codebooks || !shard_norms || !shard_stats || !sel) return RVQ_ERR_ARG;
  if (cb_dtype == RVQ_F32 && !shard_operand) return RVQ_ERR_ARG;
  const void *op = cb_dtype == RVQ_BF16 ? shard_codebooks : shard_operand;
  if (!aligned16(features) || !aligned16(shard_codebooks) || !aligned16(op) || !aligned16(shard_norms) ||
      !aligned16(sel) || (residual && !aligned16(residual)))
    return RVQ_ERR_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RVQ_ERR_WORKSPACE;
  int sms = 0;
  int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  const Plan p = make_shard_plan(N, K_shard, D, sms);
  const Layout w = make_layout(N, D, p);
  if (workspace_bytes < w.total) return RVQ_ERR_WORKSPACE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *R = residual ? residual : reinterpret_cast<float *>(ws + w.R);
  __nv_bfloat16 *Rt = reinterpret_cast<__nv_bfloat16 *>(ws + w.Rt);
  float2 *rowstat = reinterpret_cast<float2 *>(ws + w.rowstat);
  float2 *cand = reinterpret_cast<float2 *>(ws + w.cand);
  int32_t *fb_list = reinterpret_cast<int32_t *>(ws + w.fb_list);
  int32_t *fb_count = reinterpret_cast<int32_t *>(ws + w.fb_count);

  // Level 0 scores the features: bf16 features are their own operand; fp32 features get a bf16
  // copy and row statistics first.  Later levels score the residual operand written by apply.
  const bool x_is_operand = l == 0 && f_dtype == RVQ_BF16;
  const int64_t row_blocks = (N * 32 + 255) / 256;
  if (l == 0 && !x_is_operand) {
    const cudaError_t e = launch_pdl(init_kernel<false, false>, dim3(static_cast<unsigned>(row_blocks)), dim3(256), 0,
                                     s, features, N, D, R, Rt, rowstat, fb_count, 0,
                                     static_cast<const int64_t *>(nullptr), int64_t(0), status);
    note_launch();
    if (e != cudaSuccess) return RVQ_ERR_CUDA;
  }
  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, x_is_operand ? features : static_cast<const void *>(Rt), N, D, BM)) return RVQ_ERR_CUDA;
  if (!make_map(&tmB, static_cast<const uint8_t *>(op) + static_cast<size_t>(l) * K_shard * D * 2, K_shard, D,
                BN))
    return RVQ_ERR_CUDA;
  const int epi = epilogue_warps(D);
  if (!gemm_attrs_ready(epi)) return RVQ_ERR_CUDA;
  GemmArgs ga;
  ga.norms = shard_norms + static_cast<size_t>(l) * K_shard;
  ga.N = N;
  ga.K = K_shard;
  ga.D = D;
  ga.U = p.U;
  ga.Tc = p.Tc;
  ga.G = p.G;
  ga.maxs = p.maxs;
  ga.cand = cand;
  ga.status = status;
  ga.zero_counter = fb_count;  // this call's count of exact shard scans
  profile_begin(s);
  const cudaError_t ge = launch_gemm(epi, p.G, s, tmA, tmB, ga);
  profile_end(s);
  note_launch();
  if (ge != cudaSuccess) return RVQ_ERR_CUDA;

  RowArgs ra;
  ra.N = N;
  ra.D = D;
  ra.K = K_shard;
  ra.L = L;
  ra.l = l;
  ra.Tc = p.Tc;
  ra.G = p.G;
  ra.maxs = p.maxs;
  ra.U = p.U;
  ra.rt0 = 0;
  ra.nslots = 0;
  ra.cand = cand;
  ra.rowstat = rowstat;
  ra.R = R;
  ra.Rt = Rt;
  ra.cb = shard_codebooks;
  ra.stats = shard_stats + static_cast<size_t>(l) * RVQ_LEVEL_STATS;
  ra.ids = nullptr;
  ra.fb_list = fb_list;
  ra.fb_count = fb_count;
  ra.status = status;
  ra.last = l == L - 1;
  ra.src = l == 0 ? features : static_cast<const void *>(R);
  ra.fb_next = nullptr;
  ra.offsets = nullptr;
  ra.B = 0;
  double2 *sel2 = reinterpret_cast<double2 *>(sel);
  const int nch = row_chunks(D);
  const unsigned rb = static_cast<unsigned>(row_blocks), fb = static_cast<unsigned>(2 * sms);
  const bool cbb = cb_dtype == RVQ_BF16;
  cudaError_t e;
  if (l > 0)
    e = cbb ? launch_shard_select<true, SRC_R>(ra, k0, sel2, nch, rb, fb, s)
            : launch_shard_select<false, SRC_R>(ra, k0, sel2, nch, rb, fb, s);
  else if (f_dtype == RVQ_BF16)
    e = cbb ? launch_shard_select<true, SRC_X_BF16>(ra, k0, sel2, nch, rb, fb, s)
            : launch_shard_select<false, SRC_X_BF16>(ra, k0, sel2, nch, rb, fb, s);
  else
    e = cbb ? launch_shard_select<true, SRC_X_F32>(ra, k0, sel2, nch, rb, fb, s)
            : launch_shard_select<false, SRC_X_F32>(ra, k0, sel2, nch, rb, fb, s);
  note_launch(2);
  if (e != cudaSuccess) return RVQ_ERR_CUDA;
  if (fallbacks && cudaMemcpyAsync(fallbacks + l, fb_count, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return RVQ_ERR_CUDA;
  return RVQ_OK;
}

extern "C" int rvq_shard_apply(const void *features, int f_dtype, int64_t N, int D, const double *sel_all, int W,
                               const void *const *shard_codebooks, int cb_dtype, const int *shard_K, int L, int l,
                               int32_t *ids, float *residual, void *workspace, size_t workspace_bytes,
                               int32_t *status, void *stream) {
  RVQ_ENTRY("rvq_shard_apply");
  using namespace rvq;
  using namespace rvq::enc;
  if (N < 0 || D < 1 || L < 1 || l < 0 || l >= L || W < 1) return RVQ_ERR_ARG;
  if ((f_dtype != RVQ_F32 && f_dtype != RVQ_BF16) || (cb_dtype != RVQ_F32 && cb_dtype != RVQ_BF16))
    return RVQ_ERR_ARG;
  if (!shard_width_ok(D) || L > 64 || N >= (int64_t(1) << 31) || W > RVQ_MAX_SHARDS) return RVQ_ERR_UNSUPPORTED;
  if (!shard_codebooks || !shard_K) return RVQ_ERR_ARG;
  ShardApplyArgs sa = {};
  int64_t k = 0;
  for (int r = 0; r < W; ++r) {
    if (!shard_codebooks[r] || !aligned16(shard_codebooks[r]) || shard_K[r] < 1) return RVQ_ERR_ARG;
    sa.cb[r] = shard_codebooks[r];
    sa.Kw[r] = shard_K[r];
    sa.k0[r] = k;
    k += shard_K[r];
  }
  if (k >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  if (N == 0) return RVQ_OK;
  if (!features || !sel_all || !ids || !aligned16(features) || !aligned16(sel_all) ||
      (residual && !aligned16(residual)) || (reinterpret_cast<uintptr_t>(ids) & 3u))
    return RVQ_ERR_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RVQ_ERR_WORKSPACE;
  if (workspace_bytes < row_state_bytes(N, D)) return RVQ_ERR_WORKSPACE;
  sa.sel = reinterpret_cast<const double2 *>(sel_all);
  sa.W = W;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  RowArgs ra = {};
  ra.N = N;
  ra.D = D;
  ra.K = static_cast<int>(k);
  ra.L = L;
  ra.l = l;
  ra.R = residual ? residual : reinterpret_cast<float *>(ws);
  ra.Rt = reinterpret_cast<__nv_bfloat16 *>(ws + align256(static_cast<size_t>(N) * D * 4));
  ra.rowstat = reinterpret_cast<float2 *>(ws + align256(static_cast<size_t>(N) * D * 4) +
                                          align256(static_cast<size_t>(N) * D * 2));
  ra.ids = ids;
  ra.status = status;
  ra.last = l == L - 1;
  ra.src = l == 0 ? features : static_cast<const void *>(ra.R);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nch = row_chunks(D);
  const unsigned rb = static_cast<unsigned>((N * 32 + 255) / 256);
  const bool cbb = cb_dtype == RVQ_BF16;
  cudaError_t e;
  if (l > 0)
    e = cbb ? launch_shard_apply<true, SRC_R>(ra, sa, nch, rb, s) : launch_shard_apply<false, SRC_R>(ra, sa, nch, rb, s);
  else if (f_dtype == RVQ_BF16)
    e = cbb ? launch_shard_apply<true, SRC_X_BF16>(ra, sa, nch, rb, s)
            : launch_shard_apply<false, SRC_X_BF16>(ra, sa, nch, rb, s);
  else
    e = cbb ? launch_shard_apply<true, SRC_X_F32>(ra, sa, nch, rb, s)
            : launch_shard_apply<false, SRC_X_F32>(ra, sa, nch, rb, s);
  note_launch();
  return e == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}
