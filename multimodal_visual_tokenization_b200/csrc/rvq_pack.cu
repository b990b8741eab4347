// rvq_pack.cu -- packing pretokenized image sequences for data-parallel ranks (LongCat-2.5
// technical blog, "Offline Visual Preprocessing" and "Supernode-Aware Parallelism": the tokenizer
// is fixed, so the ids are computed once and cached, and because every image's token count is then
// known when batches are packed, the modality load can be kept even across data-parallel ranks).
//
//  * rvq_balance_sequences (host): longest-processing-time-first assignment of sequences to ranks
//    by token count, with fixed tie rules so every rank computes the same assignment.
//  * rvq_gather_sequences (GPU): copies the id rows of the selected sequences out of the id cache
//    into one packed [tokens, L] buffer; each selected sequence is split over gridDim.y blocks (so
//    a batch of a few dozen images still fills every SM), 16-byte copies where the rows allow it.
//    Bandwidth-bound: each id byte is read and written once.
#include <algorithm>
#include <numeric>
#include <vector>

#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {

// Copy cache rows [src0, src0 + len) to out rows [dst0, dst0 + len), L ints each, for selected
// sequence blockIdx.x (this block: piece blockIdx.y of gridDim.y); the packed length must match
// the cached one.
__global__ void __launch_bounds__(256) gather_sequences_kernel(const int32_t *__restrict__ cache, int L,
                                                               const int64_t *__restrict__ cache_offsets, int64_t S,
                                                               const int64_t *__restrict__ select,
                                                               const int64_t *__restrict__ out_offsets,
                                                               int32_t *__restrict__ out, int32_t *status) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t m = blockIdx.x;
  const int64_t s = select[m];
  if (s < 0 || s >= S) {
    if (threadIdx.x == 0) set_status(status, RVQ_ERR_ARG);
    return;
  }
  const int64_t src0 = cache_offsets[s], len = cache_offsets[s + 1] - src0;
  const int64_t dst0 = out_offsets[m];
  if (len < 0 || out_offsets[m + 1] - dst0 != len) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_status(status, RVQ_ERR_ARG);
    return;
  }
  const int32_t *src = cache + src0 * L;
  int32_t *dst = out + dst0 * L;
  const int64_t n = len * L;
  const int64_t tid = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.y) * blockDim.x;
  // 16-byte moves when both ends are 16-byte aligned, else 4-byte ones
  if (((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) == 0) {
    const int64_t n4 = n / 4;
    const int4 *s4 = reinterpret_cast<const int4 *>(src);
    int4 *d4 = reinterpret_cast<int4 *>(dst);
    for (int64_t i = tid; i < n4; i += nthreads) d4[i] = __ldcs(s4 + i);
    for (int64_t i = n4 * 4 + tid; i < n; i += nthreads) dst[i] = src[i];
  } else {
    for (int64_t i = tid; i < n; i += nthreads) dst[i] = src[i];
  }
}

}  // namespace rvq

extern "C" int rvq_balance_sequences(const int64_t *lengths, int64_t S, int world, int32_t *owner, int64_t *load) {
  RVQ_ENTRY("rvq_balance_sequences");
  using namespace rvq;
  if (S < 0 || world < 1 || !owner || !load || (S > 0 && !lengths)) return RVQ_ERR_ARG;
  for (int64_t s = 0; s < S; ++s)
    if (lengths[s] < 0) return RVQ_ERR_ARG;
  std::vector<int64_t> order(static_cast<size_t>(S));
  std::iota(order.begin(), order.end(), int64_t(0));
  // decreasing length, equal lengths in index order
  std::stable_sort(order.begin(), order.end(), [&](int64_t a, int64_t b) { return lengths[a] > lengths[b]; });
  // least loaded rank first, equal loads: lower rank (a heap of (load, rank) pairs)
  std::vector<std::pair<int64_t, int>> heap(static_cast<size_t>(world));
  for (int r = 0; r < world; ++r) heap[r] = {0, r};
  auto later = [](const std::pair<int64_t, int> &a, const std::pair<int64_t, int> &b) { return a > b; };
  std::make_heap(heap.begin(), heap.end(), later);
  for (int64_t s : order) {
    std::pop_heap(heap.begin(), heap.end(), later);
    auto &top = heap.back();
    owner[s] = top.second;
    top.first += lengths[s];
    std::push_heap(heap.begin(), heap.end(), later);
  }
  for (const auto &h : heap) load[h.second] = h.first;
  return RVQ_OK;
}

extern "C" int rvq_gather_sequences(const int32_t *cache_ids, int L, const int64_t *cache_offsets, int64_t S,
                                    const int64_t *select, int64_t M, const int64_t *out_offsets, int32_t *out_ids,
                                    int32_t *status, void *stream) {
  RVQ_ENTRY("rvq_gather_sequences");
  using namespace rvq;
  if (L < 1 || S < 0 || M < 0) return RVQ_ERR_ARG;
  if (M == 0) return RVQ_OK;
  if (M > 0x7FFFFFFF) return RVQ_ERR_UNSUPPORTED;
  if (!cache_ids || !cache_offsets || !select || !out_offsets || !out_ids) return RVQ_ERR_ARG;
  int sms = 0;
  const int st = device_sm_count(&sms);
  if (st != RVQ_OK) return st;
  // pieces per sequence: about eight blocks per SM over the whole batch
  const int pieces = static_cast<int>(std::min<int64_t>(64, std::max<int64_t>(1, (8LL * sms + M - 1) / M)));
  const cudaError_t e = launch_pdl(gather_sequences_kernel, dim3(static_cast<unsigned>(M), pieces), dim3(256), 0,
                                   static_cast<cudaStream_t>(stream), cache_ids, L, cache_offsets, S, select,
                                   out_offsets, out_ids, status);
  note_launch();
  return e == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}
