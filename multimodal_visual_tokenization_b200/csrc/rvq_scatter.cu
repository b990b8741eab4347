// rvq_scatter.cu -- row scatter-adds: the table gradient of the backbone's visual-token embedding
// (rvq_embed_backward) and the k-means update of a codebook level (rvq_codebook_update).
//
// Embedding gradient: the gradient of the backbone's visual-token embedding with respect to its tables
// (LongCat-2.5 technical blog, "Visual Primitive Modeling": the visual codebook embeddings are
// learned jointly with the backbone).  The embedding of a token is the decode gather-sum with
// learned tables, e[n] = sum_l E_l[ids[n,l]] (rvq_decode computes it); its table gradient is the
// scatter-add
//     grad[l, ids[n,l], :] += g[n, :]      for every row n and level l.
//
// Schedule: the H axis is cut into slices of 32 lanes x 4 fp32 = 128 columns and the grid runs
// slice-major, so while one slice is accumulated only L x K x 128 x 4 bytes of the gradient are
// live (64 MiB for 8 x 16384 rows) and they stay in L2; g is streamed from HBM once.  A warp
// walks rows of its slice, fetching the next row's ids while the current row's additions are in
// flight, and adds its 128 columns into the row's L destinations with 16-byte vector atomics
// (fp32x4 reductions at L2).  The order in which a destination row receives its terms is
// whatever the atomics make it, so the fp32 result can differ between runs by rounding, within
// (count - 1) * 2^-24 * sum of |terms| per element.
//
// Bound: the L2 performs the N x L x H fp32 additions as read-modify-writes (32 GiB for 2^20 rows,
// 8 levels, H = 1024) at ~3.2 TB/s on B200 (measured: 10.1 ms; bulk TMA reductions of whole
// 512-byte slices instead of fp32x4 atomics ran at the same speed), far above the time to stream g
// once.
#include <algorithm>

#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {

constexpr int kEmbedWarps = 8;
constexpr int kEmbedBlocksPerSm = 4;

__global__ void __launch_bounds__(kEmbedWarps * 32, kEmbedBlocksPerSm)
    embed_backward_kernel(const int32_t *__restrict__ ids, int64_t N, int L, int K, int H,
                          const float *__restrict__ g, float *grad, int32_t *counts, int32_t *status) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kEmbedWarps;
  int64_t n = static_cast<int64_t>(blockIdx.x) * kEmbedWarps + (threadIdx.x >> 5);
  if (n >= N) return;  // whole warp
  const int col = blockIdx.y * 128 + lane * 4;
  const bool active = col < H;
  // lane j holds the ids of levels j and j + 32 of the current row
  int id0 = lane < L ? __ldg(ids + n * L + lane) : 0;
  int id1 = lane + 32 < L ? __ldg(ids + n * L + lane + 32) : 0;
  bool bad = false;
  while (true) {
    const float4 v = active ? __ldcs(reinterpret_cast<const float4 *>(g + n * H + col)) : make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t nn = n + stride;
    const int nid0 = (lane < L && nn < N) ? __ldg(ids + nn * L + lane) : 0;
    const int nid1 = (lane + 32 < L && nn < N) ? __ldg(ids + nn * L + lane + 32) : 0;
    for (int l = 0; l < L; ++l) {
      const int id = __shfl_sync(0xffffffffu, l < 32 ? id0 : id1, l & 31);
      const bool ok = static_cast<unsigned>(id) < static_cast<unsigned>(K);
      bad |= !ok;
      if (ok && active) atomicAdd(reinterpret_cast<float4 *>(grad + (static_cast<int64_t>(l) * K + id) * H + col), v);
      if (ok && counts && lane == 0 && blockIdx.y == 0) atomicAdd(counts + static_cast<int64_t>(l) * K + id, 1);
    }
    if (nn >= N) break;
    n = nn;
    id0 = nid0;
    id1 = nid1;
  }
  if (bad && lane == 0 && blockIdx.y == 0) set_status(status, RVQ_ERR_ID_RANGE);
}

// k-means finalize: new[k] = sums[k] / count[k] (divided in fp64, rounded to fp32), or old[k] when the
// cluster is empty; one thread per 4 columns.  new may be old (each element is read before it is
// written, by the same thread).
__global__ void __launch_bounds__(256) kmeans_finalize_kernel(const float *sums, const int32_t *counts, int K, int D,
                                                              const float *old_cb, float *new_cb) {
  griddep_launch_dependents();
  griddep_wait();
  const int q = D / 4;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<int64_t>(K) * q) return;
  const int64_t k = t / q;
  const int c = counts[k];
  float4 v;
  if (c == 0) {
    v = reinterpret_cast<const float4 *>(old_cb)[t];
  } else {
    v = reinterpret_cast<const float4 *>(sums)[t];
    const double dc = static_cast<double>(c);  // exact for every count, unlike an fp32 copy above 2^24
    v.x = static_cast<float>(static_cast<double>(v.x) / dc);
    v.y = static_cast<float>(static_cast<double>(v.y) / dc);
    v.z = static_cast<float>(static_cast<double>(v.z) / dc);
    v.w = static_cast<float>(static_cast<double>(v.w) / dc);
  }
  reinterpret_cast<float4 *>(new_cb)[t] = v;
}

int launch_scatter(const int32_t *ids, int64_t N, int L, int K, int H, const float *g, float *grad, int32_t *counts,
                   int32_t *status, cudaStream_t s) {
  int sms = 0;
  const int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  const int64_t gx = std::min<int64_t>((N + kEmbedWarps - 1) / kEmbedWarps,
                                       static_cast<int64_t>(sms) * kEmbedBlocksPerSm);
  const int64_t gy = (H + 127) / 128;
  if (gy > 65535) return RVQ_ERR_UNSUPPORTED;
  const cudaError_t e = launch_pdl(embed_backward_kernel, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                                   dim3(kEmbedWarps * 32), 0, s, ids, N, L, K, H, g, grad, counts, status);
  note_launch();
  return e == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}

}  // namespace rvq

extern "C" int rvq_embed_backward(const int32_t *ids, int64_t N, int L, int K, int H, const float *grad_out,
                                  float *grad_tables, int32_t *status, void *stream) {
  RVQ_ENTRY("rvq_embed_backward");
  using namespace rvq;
  if (N < 0 || L < 1 || K < 1 || H < 1) return RVQ_ERR_ARG;
  if (L > 64 || H % 4 != 0) return RVQ_ERR_UNSUPPORTED;
  if (N == 0) return RVQ_OK;
  if (!ids || !grad_out || !grad_tables) return RVQ_ERR_ARG;
  if (!aligned16(grad_out) || !aligned16(grad_tables) || (reinterpret_cast<uintptr_t>(ids) & 3u)) return RVQ_ERR_ARG;
  return launch_scatter(ids, N, L, K, H, grad_out, grad_tables, nullptr, status, static_cast<cudaStream_t>(stream));
}

extern "C" int rvq_codebook_update(const float *points, const int32_t *ids, int64_t N, int D, int K,
                                   const float *old_codebook, float *new_codebook, float *sums, int32_t *counts,
                                   int32_t *status, void *stream) {
  RVQ_ENTRY("rvq_codebook_update");
  using namespace rvq;
  if (N < 0 || D < 1 || K < 1) return RVQ_ERR_ARG;
  if (D % 4 != 0 || N >= (int64_t(1) << 31)) return RVQ_ERR_UNSUPPORTED;
  if (!old_codebook || !new_codebook || !sums || !counts || (N > 0 && (!points || !ids))) return RVQ_ERR_ARG;
  if ((N > 0 && !aligned16(points)) || !aligned16(old_codebook) || !aligned16(new_codebook) || !aligned16(sums) ||
      (reinterpret_cast<uintptr_t>(counts) & 3u) || (N > 0 && (reinterpret_cast<uintptr_t>(ids) & 3u)))
    return RVQ_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(sums, 0, static_cast<size_t>(K) * D * sizeof(float), s) != cudaSuccess ||
      cudaMemsetAsync(counts, 0, static_cast<size_t>(K) * sizeof(int32_t), s) != cudaSuccess)
    return RVQ_ERR_CUDA;
  if (N > 0) {
    const int st = launch_scatter(ids, N, 1, K, D, points, sums, counts, status, s);
    if (st != RVQ_OK) return st;
  }
  const int64_t threads = static_cast<int64_t>(K) * (D / 4);
  const cudaError_t e = launch_pdl(kmeans_finalize_kernel, dim3(static_cast<unsigned>((threads + 255) / 256)),
                                   dim3(256), 0, s, sums, counts, K, D, old_codebook, new_codebook);
  note_launch();
  return e == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}
