// rvq_segsum.cu -- deterministic table gradient of the backbone's visual-token embedding:
//     grad[l, k, :] += sum of g[n, :] over the tokens n with ids[n, l] == k
// (LongCat-2.5 technical blog, "Visual Primitive Modeling": the visual codebook embeddings are
// learned jointly with the backbone; the forward e[n] = sum_l E_l[ids[n,l]] is rvq_decode).
//
// Instead of one fp32 atomic per (token, level, column) (rvq_embed_backward, bound by the L2's
// read-modify-write rate), the tokens of every level are sorted by id and each gradient row is
// summed by one warp and written once:
//   1. ss_hist_kernel     per (level, chunk of SS_CH tokens): histogram of the ids in shared memory
//   2. ss_prefix_kernel   per (level, id): the id's count in earlier chunks (so a chunk knows where
//                         its tokens of that id go) and its total
//   3. ss_scan_kernel     per level: segment starts (prefix sums of the totals), the list of
//                         non-empty ids and the "hot" ids (more than SS_HOT tokens) with their
//                         pieces of SS_HOT positions
//   4. ss_scatter_kernel  per (level, chunk), one warp: tokens in ascending n go to their slots
//                         (ranks among equal ids from __match_any_sync), so each segment lists its
//                         tokens in ascending n: a stable counting sort
//   5. ss_rowsum_kernel   one warp per (level, segment) or hot piece: the segment's g rows, whole
//                         (512-byte gathers per instruction), through a per-warp cp.async ring of
//                         SS_RROWS rows, summed in ascending position order and added into the
//                         gradient row with float4 atomics (the only write of those elements, so no
//                         ordering question arises); a hot id's pieces go to scratch rows instead
//   6. ss_fix_kernel      per hot id: its pieces summed in order and added into the gradient row
// Every gradient element is written by one thread, with its terms added in an order fixed by the
// ids alone, so the result is bit-identical from run to run.  Every g row is read once per level
// (L x N x H x 4 bytes, from HBM: the rows a level visits are in id order, not in memory order).
// Measured on 2^20 tokens x 8 levels x 1024 columns (level 0 Zipf(1.1), others uniform): 5.99 ms,
// against 8.97 ms for a slice-major variant that summed 64-column slices of g (so that a slice could
// stay in L2 across the level passes; 32-column slices 10.9 ms, 16 -> 21.9, 8 -> 44.3: each gather
// instruction then touched a line per lane group) and 10.1 ms for the atomic kernel.
#include <algorithm>

#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {
namespace ss {

constexpr int SS_CH = 8192;    // tokens per histogram / scatter block
constexpr int SS_PAD = 4;      // piece rows (carry) are padded to a multiple of this many columns
constexpr int SS_HOT = 256;    // segments longer than this are summed in pieces of this size
constexpr int SS_WARPS = 8;    // warps per block of the fix kernel
constexpr int SCAN_THREADS = 1024;
constexpr int MAX_K = 49151;   // K + 1 histogram counters in <= 192 KiB of shared memory

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__device__ __forceinline__ void cp_async16(float4 *dst, const float *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

struct Layout {
  int64_t nch, maxp, Hpad;
  size_t hist, start, perm, nz_key, nz_start, hot_key, hot_p0, meta, carry, total;
};

inline Layout make_layout(int64_t N, int L, int K, int H) {
  Layout w;
  w.nch = (N + SS_CH - 1) / SS_CH;
  w.maxp = std::max<int64_t>(1, 2 * ((N + SS_HOT - 1) / SS_HOT));
  w.Hpad = (H + SS_PAD - 1) / SS_PAD * SS_PAD;
  size_t off = 0;
  w.hist = off;      // [L][nch][K+1]: counts, then the id's count in earlier chunks
  off += align256(static_cast<size_t>(L) * w.nch * (K + 1) * 4);
  w.start = off;     // [L][K+1]: tokens per id, then the id's segment start
  off += align256(static_cast<size_t>(L) * (K + 1) * 4);
  w.perm = off;      // [L][N]: tokens sorted by id (ascending n within an id)
  off += align256(static_cast<size_t>(L) * N * 4);
  w.nz_key = off;    // [L][K+2]: non-empty ids in ascending order (K = out-of-range ids)
  off += align256(static_cast<size_t>(L) * (K + 2) * 4);
  w.nz_start = off;  // [L][K+2]: their segment starts, then N
  off += align256(static_cast<size_t>(L) * (K + 2) * 4);
  w.hot_key = off;   // [L][K+1]: nz index of every hot segment
  off += align256(static_cast<size_t>(L) * (K + 1) * 4);
  w.hot_p0 = off;    // [L][K+2]: first piece of every hot segment, then the piece count
  off += align256(static_cast<size_t>(L) * (K + 2) * 4);
  w.meta = off;      // [L][4]: non-empty segments, hot segments, pieces
  off += align256(static_cast<size_t>(L) * 4 * 4);
  w.carry = off;     // [L][maxp][Hpad] fp32: piece sums
  off += align256(static_cast<size_t>(L) * w.maxp * w.Hpad * 4);
  w.total = off;
  return w;
}

struct Args {
  const int32_t *ids;
  int64_t N;
  int L, K, H;
  int64_t nch, maxp, Hpad;
  int32_t *hist, *start, *perm, *nz_key, *nz_start, *hot_key, *hot_p0, *meta;
  float *carry;
  const float *g;
  float *grad;
  int32_t *status;
};

__device__ __forceinline__ int key_of(const Args &a, int64_t n, int l, bool &bad) {
  const int id = __ldg(a.ids + n * a.L + l);
  const bool ok = static_cast<unsigned>(id) < static_cast<unsigned>(a.K);
  bad |= !ok;
  return ok ? id : a.K;
}

__global__ void __launch_bounds__(512) ss_hist_kernel(const Args a) {
  extern __shared__ int cnt[];
  griddep_launch_dependents();
  griddep_wait();
  const int c = blockIdx.x, l = blockIdx.y;
  for (int k = threadIdx.x; k <= a.K; k += blockDim.x) cnt[k] = 0;
  __syncthreads();
  const int64_t n0 = static_cast<int64_t>(c) * SS_CH, n1 = min(a.N, n0 + SS_CH);
  bool bad = false;
  for (int64_t n = n0 + threadIdx.x; n < n1; n += blockDim.x) atomicAdd(&cnt[key_of(a, n, l, bad)], 1);
  if (bad) set_status(a.status, RVQ_ERR_ID_RANGE);
  __syncthreads();
  int32_t *h = a.hist + (static_cast<int64_t>(l) * a.nch + c) * (a.K + 1);
  for (int k = threadIdx.x; k <= a.K; k += blockDim.x) h[k] = cnt[k];
}

// Per (level, id): counts of the earlier chunks replace the chunk counts; the total goes to start.
__global__ void __launch_bounds__(256) ss_prefix_kernel(const Args a) {
  griddep_launch_dependents();
  griddep_wait();
  const int l = blockIdx.y;
  const int nk = a.K + 1;
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= nk) return;
  int32_t *hist = a.hist + static_cast<int64_t>(l) * a.nch * nk + k;
  int r = 0;
  for (int64_t c = 0; c < a.nch; c += 8) {  // eight chunks' counts in flight at a time
    int o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] = c + u < a.nch ? hist[(c + u) * nk] : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (c + u < a.nch) hist[(c + u) * nk] = r;
      r += o[u];
    }
  }
  a.start[static_cast<int64_t>(l) * nk + k] = r;
}

// Exclusive prefix sum over the block (blockDim.x == SCAN_THREADS); *total gets the block sum.
__device__ __forceinline__ int64_t block_scan(int64_t v, int64_t *sh, int64_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();  // sh may still be read by a previous call
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int64_t s = lane < SCAN_THREADS / 32 ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sh[lane] = s;  // inclusive prefix of warp sums
  }
  __syncthreads();
  *total = sh[SCAN_THREADS / 32 - 1];
  return (warp > 0 ? sh[warp - 1] : 0) + x - v;
}

// One block per level: segment starts, the non-empty ids and the hot ids with their pieces.
__global__ void __launch_bounds__(SCAN_THREADS) ss_scan_kernel(const Args a) {
  __shared__ int64_t sh[32];
  griddep_launch_dependents();
  griddep_wait();
  const int l = blockIdx.x;
  const int nk = a.K + 1;
  int32_t *start = a.start + static_cast<int64_t>(l) * nk;
  const int kpt = (nk + SCAN_THREADS - 1) / SCAN_THREADS;
  const int k0 = min(nk, static_cast<int>(threadIdx.x) * kpt), k1 = min(nk, k0 + kpt);
  int64_t tok = 0, nz = 0, hot = 0, pieces = 0;
  for (int k = k0; k < k1; ++k) {
    const int t = start[k];
    tok += t;
    nz += t > 0;
    if (k < a.K && t > SS_HOT) {
      ++hot;
      pieces += (t + SS_HOT - 1) / SS_HOT;
    }
  }
  int64_t tot_tok, tot_nz, tot_hot, tot_pieces;
  int64_t run = block_scan(tok, sh, &tot_tok);
  int64_t z = block_scan(nz, sh, &tot_nz);
  int64_t h = block_scan(hot, sh, &tot_hot);
  int64_t p = block_scan(pieces, sh, &tot_pieces);
  int32_t *nz_key = a.nz_key + static_cast<int64_t>(l) * (a.K + 2);
  int32_t *nz_start = a.nz_start + static_cast<int64_t>(l) * (a.K + 2);
  int32_t *hot_key = a.hot_key + static_cast<int64_t>(l) * (a.K + 1);
  int32_t *hot_p0 = a.hot_p0 + static_cast<int64_t>(l) * (a.K + 2);
  for (int k = k0; k < k1; ++k) {
    const int t = start[k];
    start[k] = static_cast<int32_t>(run);
    if (t > 0) {
      nz_key[z] = k;
      nz_start[z] = static_cast<int32_t>(run);
      if (k < a.K && t > SS_HOT) {
        hot_key[h] = static_cast<int32_t>(z);
        hot_p0[h] = static_cast<int32_t>(p);
        p += (t + SS_HOT - 1) / SS_HOT;
        ++h;
      }
      ++z;
    }
    run += t;
  }
  if (threadIdx.x == 0) {
    nz_start[tot_nz] = static_cast<int32_t>(a.N);
    hot_p0[tot_hot] = static_cast<int32_t>(tot_pieces);
    int32_t *m = a.meta + 4 * l;
    m[0] = static_cast<int32_t>(tot_nz);
    m[1] = static_cast<int32_t>(tot_hot);
    m[2] = static_cast<int32_t>(tot_pieces);
  }
}

__global__ void __launch_bounds__(32) ss_scatter_kernel(const Args a) {
  extern __shared__ int ctr[];
  griddep_launch_dependents();
  griddep_wait();
  const int c = blockIdx.x, l = blockIdx.y, lane = threadIdx.x;
  const int nk = a.K + 1;
  const int32_t *before = a.hist + (static_cast<int64_t>(l) * a.nch + c) * nk;
  const int32_t *start = a.start + static_cast<int64_t>(l) * nk;
  for (int k = lane; k < nk; k += 32) ctr[k] = start[k] + before[k];
  __syncwarp();
  int32_t *perm = a.perm + static_cast<int64_t>(l) * a.N;
  const int64_t n0 = static_cast<int64_t>(c) * SS_CH, n1 = min(a.N, n0 + SS_CH);
  bool bad = false;
  for (int64_t nb = n0; nb < n1; nb += 256) {
    int key[8];  // the ids of the next 8 steps, loaded together
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t n = nb + 32 * u + lane;
      key[u] = n < n1 ? key_of(a, n, l, bad) : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const unsigned peers = __match_any_sync(0xffffffffu, key[u]);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = key[u] >= 0 ? ctr[key[u]] + rank : 0;
      __syncwarp();
      if (key[u] >= 0) {
        perm[pos] = static_cast<int32_t>(nb + 32 * u + lane);
        if (rank == 0) ctr[key[u]] += __popc(peers);
      }
      __syncwarp();
    }
  }
}

// The sum: one warp per (level, non-empty segment) or hot piece, over all H columns in passes of
// SS_RCOLS (lane j holds columns 128 q + 4 j .. + 3 of the pass, q = 0 .. 7), so every gather
// instruction moves 512 contiguous bytes of one g row.  g rows come in through a per-warp cp.async
// ring of SS_RROWS rows; each lane reads back only the 16-byte pieces it copied itself.  The terms
// of every element are added in ascending positions of its segment, starting from zero.
constexpr int SS_RWARPS = 4;    // warps per block
constexpr int SS_RROWS = 6;     // g rows in flight per warp
constexpr int SS_RCOLS = 1024;  // columns per pass: 32 lanes x 8 float4
constexpr int SS_RSMEM = SS_RWARPS * SS_RROWS * SS_RCOLS * 4;

__global__ void __launch_bounds__(SS_RWARPS * 32) ss_rowsum_kernel(const Args a, int64_t units_per_level,
                                                                   int64_t seg_units) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t wg = static_cast<int64_t>(blockIdx.x) * SS_RWARPS + (threadIdx.x >> 5);
  const int l = static_cast<int>(wg / units_per_level);
  const int64_t u = wg % units_per_level;
  if (l >= a.L) return;  // whole warp
  const int32_t *perm = a.perm + static_cast<int64_t>(l) * a.N;
  const int32_t *nz_start = a.nz_start + static_cast<int64_t>(l) * (a.K + 2);
  const int32_t *m = a.meta + 4 * l;
  int64_t j0 = 0, j1 = 0;
  float *dst = nullptr;
  bool piece = false;
  if (u < seg_units) {
    if (u >= __ldg(m)) return;  // beyond the non-empty segments
    const int key = __ldg(a.nz_key + static_cast<int64_t>(l) * (a.K + 2) + u);
    j0 = __ldg(nz_start + u);
    j1 = __ldg(nz_start + u + 1);
    if (key >= a.K || j1 - j0 > SS_HOT) return;  // out-of-range ids, or a hot id (summed in pieces)
    dst = a.grad + (static_cast<int64_t>(l) * a.K + key) * a.H;
  } else {
    const int64_t pi = u - seg_units;  // piece index
    const int nhot = __ldg(m + 1), npieces = __ldg(m + 2);
    if (pi >= npieces) return;
    const int32_t *hot_p0 = a.hot_p0 + static_cast<int64_t>(l) * (a.K + 2);
    int lo = 0, hi = nhot;  // last h with hot_p0[h] <= pi
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(hot_p0 + mid) <= pi) lo = mid;
      else hi = mid;
    }
    const int zi = __ldg(a.hot_key + static_cast<int64_t>(l) * (a.K + 1) + lo);
    const int64_t base = __ldg(nz_start + zi), end = __ldg(nz_start + zi + 1);
    j0 = base + (pi - __ldg(hot_p0 + lo)) * SS_HOT;
    j1 = min(end, j0 + SS_HOT);
    dst = a.carry + (static_cast<int64_t>(l) * a.maxp + pi) * a.Hpad;
    piece = true;
  }
  // tokens of the (at most SS_HOT = 256) positions: lane j holds position j0 + 32 w + j in tok[w]
  static_assert(SS_HOT <= 256, "a segment's tokens must fit the 8 windows of 32");
  int tok[8];
#pragma unroll
  for (int w = 0; w < 8; ++w) tok[w] = j0 + 32 * w + lane < j1 ? __ldg(perm + j0 + 32 * w + lane) : 0;
  auto token = [&](int64_t p) -> int {
    const int d = static_cast<int>(p - j0);
    int t = tok[0];
#pragma unroll
    for (int w = 1; w < 8; ++w)
      if ((d >> 5) == w) t = tok[w];
    return __shfl_sync(0xffffffffu, t, d & 31);
  };
  extern __shared__ float4 rring[];
  float4 *ring = rring + static_cast<int64_t>(threadIdx.x >> 5) * SS_RROWS * (SS_RCOLS / 4) + lane;
  auto add4 = [](float4 &x, const float4 &y) {
    x.x += y.x;
    x.y += y.y;
    x.z += y.z;
    x.w += y.w;
  };
  for (int c0 = 0; c0 < a.H; c0 += SS_RCOLS) {
    auto issue = [&](int64_t p) {
      const int slot = static_cast<int>((p - j0) % SS_RROWS);
      const float *src = a.g + static_cast<int64_t>(token(p)) * a.H + c0 + 4 * lane;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (c0 + 128 * q + 4 * lane < a.H) cp_async16(ring + (slot * 8 + q) * 32, src + 128 * q);
    };
#pragma unroll
    for (int r = 0; r < SS_RROWS - 1; ++r) {
      if (j0 + r < j1) issue(j0 + r);
      cp_async_commit();
    }
    float4 acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t p = j0; p < j1; ++p) {
      if (p + SS_RROWS - 1 < j1) issue(p + SS_RROWS - 1);
      cp_async_commit();
      cp_async_wait<SS_RROWS - 1>();  // position p has landed
      const int slot = static_cast<int>((p - j0) % SS_RROWS);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (c0 + 128 * q + 4 * lane < a.H) add4(acc[q], ring[(slot * 8 + q) * 32]);
    }
    cp_async_wait<0>();
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int col = c0 + 128 * q + 4 * lane;
      if (col >= a.H) continue;
      float4 *d = reinterpret_cast<float4 *>(dst + col);
      if (piece)
        *d = acc[q];
      else
        atomicAdd(d, acc[q]);  // the only write of these elements
    }
  }
}

// One warp per (level, hot id): its pieces' sums in piece order, added into the gradient row.
__global__ void __launch_bounds__(SS_WARPS * 32) ss_fix_kernel(const Args a, int hot_max) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * SS_WARPS + (threadIdx.x >> 5);
  const int l = static_cast<int>(w / hot_max);
  const int h = static_cast<int>(w % hot_max);
  if (l >= a.L || h >= __ldg(a.meta + 4 * l + 1)) return;
  const int32_t *hot_p0 = a.hot_p0 + static_cast<int64_t>(l) * (a.K + 2);
  const int zi = __ldg(a.hot_key + static_cast<int64_t>(l) * (a.K + 1) + h);
  const int k = __ldg(a.nz_key + static_cast<int64_t>(l) * (a.K + 2) + zi);
  const int p0 = __ldg(hot_p0 + h), p1 = __ldg(hot_p0 + h + 1);
  for (int col = lane * 4; col < a.H; col += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = p0; p < p1; ++p) {
      const float4 v = *reinterpret_cast<const float4 *>(a.carry + (static_cast<int64_t>(l) * a.maxp + p) * a.Hpad + col);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    float4 *d = reinterpret_cast<float4 *>(a.grad + (static_cast<int64_t>(l) * a.K + k) * a.H + col);
    float4 o = *d;
    o.x += acc.x;
    o.y += acc.y;
    o.z += acc.z;
    o.w += acc.w;
    *d = o;
  }
}

bool attrs_ready() {
  static int ok = -1;
  if (ok < 0) {
    const int bytes = (MAX_K + 1) * 4;
    ok = cudaFuncSetAttribute(ss_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
         cudaFuncSetAttribute(ss_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess &&
         cudaFuncSetAttribute(ss_rowsum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SS_RSMEM) == cudaSuccess;
  }
  return ok == 1;
}

}  // namespace ss
}  // namespace rvq

extern "C" int rvq_embed_backward_workspace_size(int64_t N, int L, int K, int H, size_t *bytes) {
  RVQ_ENTRY("rvq_embed_backward_workspace_size");
  using namespace rvq;
  if (!bytes || N < 0 || L < 1 || K < 1 || H < 1) return RVQ_ERR_ARG;
  if (L > 64 || H % 4 != 0 || K > ss::MAX_K || N >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  *bytes = ss::make_layout(N, L, K, H).total;
  return RVQ_OK;
}

extern "C" int rvq_embed_backward_sorted(const int32_t *ids, int64_t N, int L, int K, int H, const float *grad_out,
                                         float *grad_tables, void *workspace, size_t workspace_bytes,
                                         int32_t *status, void *stream) {
  RVQ_ENTRY("rvq_embed_backward_sorted");
  using namespace rvq;
  using namespace rvq::ss;
  if (N < 0 || L < 1 || K < 1 || H < 1) return RVQ_ERR_ARG;
  if (L > 64 || H % 4 != 0 || K > MAX_K || N >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  if (N == 0) return RVQ_OK;
  if (!ids || !grad_out || !grad_tables) return RVQ_ERR_ARG;
  if (!aligned16(grad_out) || !aligned16(grad_tables) || (reinterpret_cast<uintptr_t>(ids) & 3u)) return RVQ_ERR_ARG;
  const Layout w = make_layout(N, L, K, H);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < w.total)
    return RVQ_ERR_WORKSPACE;
  if (!attrs_ready()) return RVQ_ERR_CUDA;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  Args a;
  a.ids = ids;
  a.N = N;
  a.L = L;
  a.K = K;
  a.H = H;
  a.nch = w.nch;
  a.maxp = w.maxp;
  a.Hpad = w.Hpad;
  a.hist = reinterpret_cast<int32_t *>(ws + w.hist);
  a.start = reinterpret_cast<int32_t *>(ws + w.start);
  a.perm = reinterpret_cast<int32_t *>(ws + w.perm);
  a.nz_key = reinterpret_cast<int32_t *>(ws + w.nz_key);
  a.nz_start = reinterpret_cast<int32_t *>(ws + w.nz_start);
  a.hot_key = reinterpret_cast<int32_t *>(ws + w.hot_key);
  a.hot_p0 = reinterpret_cast<int32_t *>(ws + w.hot_p0);
  a.meta = reinterpret_cast<int32_t *>(ws + w.meta);
  a.carry = reinterpret_cast<float *>(ws + w.carry);
  a.g = grad_out;
  a.grad = grad_tables;
  a.status = status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t hsm = static_cast<size_t>(K + 1) * 4;
  const dim3 chunks(static_cast<unsigned>(w.nch), static_cast<unsigned>(L));
  const dim3 ids_grid(static_cast<unsigned>((K + 1 + 255) / 256), static_cast<unsigned>(L));
  if (launch_pdl(ss_hist_kernel, chunks, dim3(512), hsm, s, a) != cudaSuccess ||
      launch_pdl(ss_prefix_kernel, ids_grid, dim3(256), 0, s, a) != cudaSuccess ||
      launch_pdl(ss_scan_kernel, dim3(L), dim3(SCAN_THREADS), 0, s, a) != cudaSuccess ||
      launch_pdl(ss_scatter_kernel, chunks, dim3(32), hsm, s, a) != cudaSuccess)
    return RVQ_ERR_CUDA;
  const int64_t seg_max = std::min<int64_t>(static_cast<int64_t>(K) + 1, N);  // non-empty ids (with the bucket)
  const int hot_max = static_cast<int>(std::min<int64_t>(K, N / SS_HOT + 1));
  const int64_t fix_blocks = (static_cast<int64_t>(L) * hot_max + SS_WARPS - 1) / SS_WARPS;
  if (fix_blocks >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  const int64_t units = seg_max + w.maxp;  // per level: segments, then hot pieces
  const int64_t row_blocks = (static_cast<int64_t>(L) * units + SS_RWARPS - 1) / SS_RWARPS;
  if (row_blocks >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  if (launch_pdl(ss_rowsum_kernel, dim3(static_cast<unsigned>(row_blocks)), dim3(SS_RWARPS * 32), SS_RSMEM, s, a,
                 units, seg_max) != cudaSuccess ||
      launch_pdl(ss_fix_kernel, dim3(static_cast<unsigned>(fix_blocks)), dim3(SS_WARPS * 32), 0, s, a, hot_max) !=
          cudaSuccess)
    return RVQ_ERR_CUDA;
  note_launch(6);
  return RVQ_OK;
}
