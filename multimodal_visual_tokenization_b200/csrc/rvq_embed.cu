// rvq_embed.cu -- gradient of the backbone's visual-token embedding with respect to its tables
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
                          const float *__restrict__ g, float *grad, int32_t *status) {
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
    }
    if (nn >= N) break;
    n = nn;
    id0 = nid0;
    id1 = nid1;
  }
  if (bad && lane == 0 && blockIdx.y == 0) set_status(status, RVQ_ERR_ID_RANGE);
}

}  // namespace rvq

extern "C" int rvq_embed_backward(const int32_t *ids, int64_t N, int L, int K, int H, const float *grad_out,
                                  float *grad_tables, int32_t *status, void *stream) {
  using namespace rvq;
  if (N < 0 || L < 1 || K < 1 || H < 1) return RVQ_ERR_ARG;
  if (L > 64 || H % 4 != 0) return RVQ_ERR_UNSUPPORTED;
  if (N == 0) return RVQ_OK;
  if (!ids || !grad_out || !grad_tables) return RVQ_ERR_ARG;
  if (!aligned16(grad_out) || !aligned16(grad_tables) || (reinterpret_cast<uintptr_t>(ids) & 3u)) return RVQ_ERR_ARG;
  int sms = 0;
  const int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  const int64_t gx = std::min<int64_t>((N + kEmbedWarps - 1) / kEmbedWarps,
                                       static_cast<int64_t>(sms) * kEmbedBlocksPerSm);
  const int64_t gy = (H + 127) / 128;
  if (gy > 65535) return RVQ_ERR_UNSUPPORTED;
  const cudaError_t e = launch_pdl(embed_backward_kernel, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                                   dim3(kEmbedWarps * 32), 0, static_cast<cudaStream_t>(stream), ids, N, L, K, H,
                                   grad_out, grad_tables, status);
  note_launch();
  return e == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}
