/*
 * rvq.h -- C ABI of librvq.so: residual vector quantization (RVQ) of visual
 * features into multi-level discrete token ids, and the gather-sum decode back
 * to feature space, on one NVIDIA B200 (sm_100a).
 *
 * Method.  The LongCat-2.5 technical blog ("Visual Primitive Modeling" ->
 * "Discrete Native Resolution Vision Transformer") applies RVQ to native-
 * resolution encoder features so that an image becomes a sequence of
 * multi-level tokens; the Meituan LongCat-2.5 open-source article (section
 * "02 Visual Coding and 3D") says the quantizer adds detail level by level;
 * Figure 1 of the blog shows the ids being reconstructed by a de-tokenizer; and
 * "Offline Visual Preprocessing" fixes the tokenizer so ids are precomputed once.
 * The pages give no code, sizes or metric.  This library implements the plain
 * reading of that description: greedy RVQ under squared Euclidean distance,
 *
 *     r_0 = x;  for l in 0..L-1:  id_l = argmin_k ||r_l - C_l[k]||^2  (lowest k on ties)
 *                                 r_{l+1} = r_l - C_l[id_l]
 *     decode(ids) = sum_l C_l[id_l]           (fp32 accumulation, ascending l)
 *
 * Conventions for every entry point
 *   - All array pointers are DEVICE pointers owned by the caller, 16-byte aligned,
 *     row-major and densely packed.  The library allocates no device memory between
 *     calls except lazily created profiling events.  It does hold one statically sized
 *     array, the RVQ_NOALLOC_SCRATCH_BYTES (32 MiB) scratch of rvq_encode_noalloc, on every
 *     device where librvq.so's module is loaded, whichever entry points the caller uses.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued
 *     asynchronously; the call returns after enqueueing.
 *   - The return value is an rvq_status.  Argument errors are detected on the host
 *     before anything is enqueued (nothing is written).  Errors found on the device
 *     (an id out of range, a pipeline wait that timed out) are written to the
 *     optional caller-owned device word `*status` (0 = ok); the first error wins.
 *     Read it after synchronising the stream.
 *   - Inputs must be finite.  Calls that overlap on the GPU must not share output or
 *     workspace buffers.
 *   - Every compute entry point opens an NVTX range named after itself (visible to nsys / ncu).
 *   - Host-side fault injection, for testing a caller's error handling without a GPU fault:
 *     with RVQ_FAULT="<entry point>:<status>[,...]" in the environment (read once, at the first
 *     call), each named entry point returns that negative rvq_status at once, before it checks
 *     its arguments or touches the device.  E.g. RVQ_FAULT="rvq_encode:-4,rvq_decode:-5".
 */
#ifndef RVQ_H_
#define RVQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RVQ_API __attribute__((visibility("default")))
#else
#define RVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Storage type of features / codebooks. */
typedef enum { RVQ_F32 = 0, RVQ_BF16 = 1 } rvq_dtype;

typedef enum {
    RVQ_OK = 0,
    RVQ_ERR_ARG = -1,          /* null pointer, negative size, misaligned pointer, bad offsets */
    RVQ_ERR_UNSUPPORTED = -2,  /* shape outside the supported range (see each call) */
    RVQ_ERR_WORKSPACE = -3,    /* workspace missing or smaller than rvq_encode_workspace_size */
    RVQ_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed */
    RVQ_ERR_ID_RANGE = -5,     /* decode met an id outside [0, K) (device-detected) */
    RVQ_ERR_TIMEOUT = -6       /* an encode pipeline wait gave up (device-detected) */
} rvq_status;

/* Per-level codebook statistics written by rvq_build_norms, RVQ_LEVEL_STATS floats per level:
 *   [0] max_k ||C_l[k]||            [1] max_k ||C_l[k] - bf16(C_l[k])||
 *   [2] max_k ||bf16(C_l[k])||      [3] max_k fl32(||C_l[k]||^2)
 * (each rounded upward).  rvq_encode uses them to bound the error of its bf16 tensor-core
 * distances and so decide when a candidate list provably holds the nearest codeword. */
#define RVQ_LEVEL_STATS 4

/*
 * rvq_build_norms -- one-off preparation of a fixed codebook set ("Offline Visual
 * Preprocessing": the tokenizer is fixed, so this runs once per codebook set).
 *   codebooks    [L, K, D] in cb_dtype
 *   norms        [L, K] fp32 out: ||C_l[k]||^2 (fp32 lane sums of <= ceil(D/32) squares, combined
 *                in fp64, rounded to nearest: relative error <= (D/32+2) 2^-24)
 *   level_stats  [L, RVQ_LEVEL_STATS] fp32 out (see above)
 *   cb_operand   [L, K, D] bf16 out: round-to-nearest-even copy used as the tensor-core
 *                operand.  Required when cb_dtype == RVQ_F32; ignored (may be NULL) for
 *                RVQ_BF16, where the codebooks themselves are the operand.
 * Supported: 1 <= L <= 64, 1 <= K < 2^31, 16 <= D <= 8192 with D % 16 == 0.
 */
RVQ_API int rvq_build_norms(const void *codebooks, int cb_dtype, int L, int K, int D,
                    float *norms, float *level_stats, void *cb_operand, void *stream);

/*
 * rvq_encode_workspace_size -- bytes of device workspace rvq_encode needs for these
 * sizes on the current device.  Writes *bytes; returns an rvq_status.
 */
RVQ_API int rvq_encode_workspace_size(int64_t N, int D, int L, int K, size_t *bytes);

/*
 * rvq_encode -- greedy RVQ of N feature vectors (blog, "Discrete Native Resolution Vision
 * Transformer"; article, "02 Visual Coding and 3D": detail added level by level).
 *   features     [N, D] in f_dtype (native-resolution patch features; several images may be
 *                packed back to back)
 *   codebooks    [L, K, D] in cb_dtype; cb_operand = the bf16 copy from rvq_build_norms
 *                (NULL when cb_dtype == RVQ_BF16)
 *   norms, level_stats  from rvq_build_norms for these codebooks
 *   offsets      optional [B+1] int64 image boundaries of the packed batch (offsets[0] = 0,
 *                non-decreasing, offsets[B] = N); checked on the device, not used in the
 *                arithmetic (every row is quantized independently).  NULL with B = 0 if absent.
 *   ids          [N, L] int32 out
 *   residual     optional [N, D] fp32 out: r_L (fp32 running residual)
 *   recon        optional [N, D] fp32 out: sum_l C_l[ids_l], same arithmetic as rvq_decode
 *   fallbacks    optional [L] int32 out: per level, rows whose candidate list could not be
 *                certified and were resolved by an exact scan of all K codewords
 *   workspace    >= rvq_encode_workspace_size bytes, 256-byte aligned
 * Distances: bf16 tensor-core scores ||c||^2 - 2 r.c select up to 8 candidates per row, which
 * are rescored exactly (fp64 accumulation of fp32 differences); a row whose candidates cannot
 * be proven to contain the nearest codeword is rescanned exactly.  Ties go to the lowest id.
 * Supported: N >= 0 (N = 0 is a no-op), N < 2^31, 1 <= L <= 64, 1 <= K < 2^31, 64 <= D <= 4096 with
 * D % 64 == 0.
 */
RVQ_API int rvq_encode(const void *features, int f_dtype, int64_t N, int D,
               const void *codebooks, int cb_dtype, const void *cb_operand,
               const float *norms, const float *level_stats, int L, int K,
               const int64_t *offsets, int64_t B,
               int32_t *ids, float *residual, float *recon, int32_t *fallbacks,
               void *workspace, size_t workspace_bytes, int32_t *status, void *stream);

/*
 * rvq_encode_noalloc -- rvq_encode for callers that cannot allocate device memory.
 * No counterpart in the pages: this is a deployment variant of rvq_encode.
 *
 * Some callers may not call cudaMalloc (or any allocating routine) at the point where they
 * tokenize: code running under a framework that owns all device memory through its own pool,
 * latency-critical serving loops that must not allocate (cudaMalloc can synchronize the
 * device), or plugin hosts that hand out no workspace.  This entry point takes the same
 * arguments as rvq_encode except the workspace: its scratch lives in a statically sized
 * device array compiled into librvq.so, RVQ_NOALLOC_SCRATCH_BYTES bytes, which every GPU
 * that loads the library holds until the process exits.  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *   - Sizes whose rvq_encode_workspace_size exceeds RVQ_NOALLOC_SCRATCH_BYTES are rejected with
 *     RVQ_ERR_WORKSPACE before anything is enqueued (use rvq_encode with a workspace instead).
 *   - The first call on a device looks up the scratch array's device address with that device
 *     current (once per device, and again after the device's context was replaced, e.g. by
 *     cudaDeviceReset); make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents (the kernels
 *     initialise everything they read).  Calls that overlap on the GPU (different streams,
 *     or threads) race on it: serialise them.
 * Results are identical to rvq_encode with the same inputs.
 */
#define RVQ_NOALLOC_SCRATCH_BYTES (32u << 20)
RVQ_API int rvq_encode_noalloc(const void *features, int f_dtype, int64_t N, int D,
                       const void *codebooks, int cb_dtype, const void *cb_operand,
                       const float *norms, const float *level_stats, int L, int K,
                       const int64_t *offsets, int64_t B,
                       int32_t *ids, float *residual, float *recon, int32_t *fallbacks,
                       int32_t *status, void *stream);

/*
 * rvq_decode -- gather-sum de-tokenizer input (blog, Figure 1): recon[n] = sum_l C_l[ids[n,l]],
 * fp32 accumulation in ascending l.
 *   ids      [N, L] int32;  codebooks [L, K, D] in cb_dtype;  recon [N, D] fp32 out
 * An id outside [0, K) contributes nothing and sets *status = RVQ_ERR_ID_RANGE.
 * Supported: N >= 0, 1 <= L <= 64, 1 <= K < 2^31, 4 <= D with D % 4 == 0.
 */
RVQ_API int rvq_decode(const int32_t *ids, int64_t N, int L, const void *codebooks, int cb_dtype,
               int K, int D, float *recon, int32_t *status, void *stream);

/*
 * rvq_decode_slice_plan: how rvq_decode splits the work for this shape (host only, no device
 * call).  A warp walks the rows of one column slice of `*slice_cols` columns with
 * `*rows_per_warp` rows at a time (32 / rows_per_warp lanes per row); the slice narrows (2 or 4
 * rows per warp) when its live codebook columns, L * K * slice_cols * element size, would exceed
 * 64 MiB of L2.  Same argument checks as rvq_decode (RVQ_ERR_ARG for null outputs).
 */
RVQ_API int rvq_decode_slice_plan(int L, int K, int D, int cb_dtype, int *rows_per_warp, int *slice_cols);

/* Human-readable name of an rvq_status value (static string). */
RVQ_API const char *rvq_status_str(int status);

/*
 * rvq_embed_backward -- gradient of the backbone's visual-token embedding with respect to its
 * tables (LongCat-2.5 technical blog, "Visual Primitive Modeling": the visual codebook embeddings
 * are learned jointly with the backbone).  The embedding of token n is the decode gather-sum
 * with learned tables E [L,K,H], e[n] = sum_l E_l[ids[n,l]] (rvq_decode with the tables computes
 * it).  Given grad_out = dLoss/de [N,H] fp32 row-major, this adds, for every n and l,
 *     grad_tables[l, ids[n,l], :] += grad_out[n, :]
 * into grad_tables [L,K,H] fp32 row-major (the caller zeroes it for a fresh gradient; existing
 * values are accumulated into).  Additions into one row arrive in no fixed order (fp32 atomics),
 * so results can differ between runs by rounding, within (count - 1) * 2^-24 * sum of |terms|
 * per element.  ids [N,L] int32.  An id outside [0, K) is skipped and RVQ_ERR_ID_RANGE goes to
 * *status (optional device int32, first error wins).  All array pointers are caller-owned device
 * pointers; grad_out and grad_tables 16-byte aligned.  Asynchronous on `stream`.
 * Supported: N >= 0 (N = 0 is a no-op), 1 <= L <= 64, 1 <= K < 2^31, H % 4 == 0, H <= 65535 * 128.
 */
RVQ_API int rvq_embed_backward(const int32_t *ids, int64_t N, int L, int K, int H, const float *grad_out,
                               float *grad_tables, int32_t *status, void *stream);

/*
 * rvq_embed_backward_sorted -- the same table gradient as rvq_embed_backward, deterministic: the
 * tokens of every level are sorted by id (a stable counting sort) and each gradient row receives
 * its terms from one thread in an order fixed by the ids alone (ascending token index; ids with
 * more than 256 tokens summed in pieces of 256 tokens, the pieces then added in ascending order),
 * so repeated calls on the same inputs give bit-identical gradients.
 * Each element still lies within (count - 1) * 2^-24 * sum of |terms| of the exact sum.
 * workspace: >= rvq_embed_backward_workspace_size bytes of device memory, 256-byte aligned
 * (RVQ_ERR_WORKSPACE otherwise); other arguments, status and id-range handling as in
 * rvq_embed_backward.  Supported: N < 2^31, 1 <= L <= 64, 1 <= K <= 49151, H % 4 == 0.
 * rvq_embed_backward_workspace_size writes the workspace bytes for these sizes into *bytes.
 */
RVQ_API int rvq_embed_backward_workspace_size(int64_t N, int L, int K, int H, size_t *bytes);
RVQ_API int rvq_embed_backward_sorted(const int32_t *ids, int64_t N, int L, int K, int H, const float *grad_out,
                                      float *grad_tables, void *workspace, size_t workspace_bytes,
                                      int32_t *status, void *stream);

/*
 * rvq_codebook_update -- one k-means (Lloyd) update of one codebook level: the step that fits the
 * fixed tokenizer whose ids the pages precompute offline (LongCat-2.5 technical blog, "Offline
 * Visual Preprocessing"; the pages do not describe the fitting: plain k-means on the level's input
 * residuals is the reading).  points [N,D] fp32 are the level's input residuals r_l (for level 0
 * the features), ids [N] int32 their assigned codewords (the level's column of rvq_encode's ids,
 * made contiguous).  For every k:
 *     counts[k] = #{n : ids[n] == k}
 *     new_codebook[k] = (sum of points[n] over those n) / counts[k]   (fp32 sum, any order)
 *     new_codebook[k] = old_codebook[k]                                (counts[k] == 0)
 * old_codebook, new_codebook [K,D] fp32 (they may be the same buffer: an in-place update); sums
 * [K,D] fp32 is caller-owned scratch; counts [K] int32 is an output.  All are caller-owned device
 * pointers, 16-byte aligned (counts, ids 4-byte).  Ids outside [0, K) are skipped and
 * RVQ_ERR_ID_RANGE goes to *status (optional device int32).  Asynchronous on `stream`.
 * Supported: 0 <= N < 2^31, D % 4 == 0, K >= 1.
 */
RVQ_API int rvq_codebook_update(const float *points, const int32_t *ids, int64_t N, int D, int K,
                                const float *old_codebook, float *new_codebook, float *sums, int32_t *counts,
                                int32_t *status, void *stream);

/*
 * Packing pretokenized image sequences for data-parallel ranks (LongCat-2.5 technical blog,
 * "Offline Visual Preprocessing" and "Supernode-Aware Parallelism": with the ids precomputed,
 * every image's token count is known when batches are packed, which keeps the load even across
 * data-parallel ranks; the pages give no algorithm).
 *
 * rvq_balance_sequences (host only, no GPU): assigns S sequences of lengths[S] (>= 0 tokens) to
 * `world` ranks, longest processing time first: sequences in decreasing length (equal lengths:
 * lower index first) each go to the least-loaded rank so far (equal loads: lower rank), so every
 * rank computes the same assignment from the same lengths.  owner[S] receives the rank of each
 * sequence, load[world] each rank's total tokens; the largest load is at most
 * (4/3 - 1/(3 world)) times the best possible.  Host pointers.  RVQ_ERR_ARG on bad arguments.
 *
 * rvq_gather_sequences (GPU): packs the id rows of M selected sequences out of an id cache.
 * cache_ids [T, L] int32 holds the ids of all cached sequences back to back, sequence s being rows
 * [cache_offsets[s], cache_offsets[s+1]) (cache_offsets [S+1], int64); select [M] int64 lists the
 * sequences to pack; out_offsets [M+1] int64 gives where each lands in out_ids [out_offsets[M], L]
 * (prefix sums of the selected lengths, computed by the caller, who knows them from the balance).
 * A selected index outside [0, S) or an out_offsets span that differs from the cached length is
 * skipped and RVQ_ERR_ARG goes to *status (optional device int32).  All array pointers are
 * caller-owned device pointers.  Asynchronous on `stream`.  Supported: M < 2^31.
 */
RVQ_API int rvq_balance_sequences(const int64_t *lengths, int64_t S, int world, int32_t *owner, int64_t *load);
RVQ_API int rvq_gather_sequences(const int32_t *cache_ids, int L, const int64_t *cache_offsets, int64_t S,
                                 const int64_t *select, int64_t M, const int64_t *out_offsets, int32_t *out_ids,
                                 int32_t *status, void *stream);

/*
 * Codebook-sharded encode: the same greedy RVQ as rvq_encode, with the codebook axis split over W
 * ranks (one process per GPU) for codebook sets larger than one GPU holds.  The pages only fix the
 * quantizer (LongCat-2.5 technical blog, "Discrete Native Resolution Vision Transformer": residual
 * levels of nearest codewords); the split is this library's.  Rank w holds codewords
 * [k0_w, k0_w + K_w) of every level, k0_w = K_0 + ... + K_{w-1}, as its own [L, K_w, D] array with
 * norms / level statistics / operand copy from rvq_build_norms on that array, and every rank holds
 * all N feature rows.  Per level l, in this order on every rank:
 *   1. rvq_shard_select: this shard's nearest codeword for every row, with its exact distance,
 *      into sel [N, 2] fp64 = (||r - c||^2 as an fp64 sum of fp32 differences, global id).  Same
 *      candidate / certificate / exact-rescan scheme as rvq_encode, restricted to the shard.
 *   2. the caller gathers every rank's sel into sel_all [W, N, 2] (rank w's at row block w), e.g.
 *      an all-gather over the ranks' process group.
 *   3. rvq_shard_apply: per row the lowest (distance, id) of sel_all is the level's id; ids[n, l]
 *      receives it and the residual is updated with that codeword, read from its owner's array.
 * The residual state lives in the workspace (or in `residual`, when given), so one rank's calls of
 * one encode share workspace and residual pointer, and every rank's state stays bit-identical.  The
 * ids equal rvq_encode's for the whole codebook set (exact distances; ties to the lowest id).
 *
 * rvq_shard_workspace_size: device bytes for this rank (N rows, width D, K_shard codewords).
 * rvq_shard_select: features [N, D] (f_dtype; read at l = 0), this rank's shard_codebooks
 *   [L, K_shard, D] in cb_dtype, shard_operand (bf16 copy, NULL for RVQ_BF16), shard_norms [L,
 *   K_shard] and shard_stats [L, RVQ_LEVEL_STATS] from rvq_build_norms of the shard; k0 = the
 *   shard's first global id; residual optional [N, D] fp32 (the residual after the level applied
 *   last); sel [N, 2] fp64 out; fallbacks optional [L] int32 device, entry l = rows of this level
 *   that needed an exact scan of the shard.  Device pointers 16-byte aligned; workspace 256-byte.
 * rvq_shard_apply: sel_all [W, N, 2] fp64; shard_codebooks = HOST array of W device pointers, entry
 *   w pointing at rank w's [L, K_w, D] stored codebooks (a pointer from rvq_ipc_import for another
 *   GPU's array); shard_K host array [W]; ids [N, L] int32 out (column l); residual as for select.
 *   A row whose sel entries are all unusable (non-finite inputs) gets id -1 and RVQ_ERR_ARG in
 *   *status.
 * Both: asynchronous on `stream`; argument errors are returned before anything is enqueued.
 * Supported: 64 <= D <= 1024, D % 64 == 0, 1 <= L <= 64, N < 2^31, 1 <= W <= RVQ_MAX_SHARDS,
 * total K < 2^31.
 */
#define RVQ_MAX_SHARDS 16
RVQ_API int rvq_shard_workspace_size(int64_t N, int D, int K_shard, size_t *bytes);
RVQ_API int rvq_shard_select(const void *features, int f_dtype, int64_t N, int D, const void *shard_codebooks,
                             int cb_dtype, const void *shard_operand, const float *shard_norms,
                             const float *shard_stats, int L, int K_shard, int64_t k0, int l, float *residual,
                             double *sel, int32_t *fallbacks, void *workspace, size_t workspace_bytes,
                             int32_t *status, void *stream);
RVQ_API int rvq_shard_apply(const void *features, int f_dtype, int64_t N, int D, const double *sel_all, int W,
                            const void *const *shard_codebooks, int cb_dtype, const int *shard_K, int L, int l,
                            int32_t *ids, float *residual, void *workspace, size_t workspace_bytes,
                            int32_t *status, void *stream);

/*
 * Device buffers shared between the processes of one node (CUDA IPC), for rvq_shard_apply's
 * peer pointers.  rvq_ipc_export: the RVQ_IPC_HANDLE_BYTES-byte handle of the device allocation
 * that holds ptr, and ptr's byte offset in it (host outputs).  rvq_ipc_import (another process):
 * maps that allocation on the current device (peer access enabled on first use) and returns
 * *ptr = its base + offset; the mapping stays valid while the exporting process keeps the
 * allocation.  rvq_ipc_close(ptr, offset) unmaps it.  RVQ_ERR_ARG for a pointer that is not
 * device memory, RVQ_ERR_CUDA when the runtime refuses (e.g. import in the exporting process).
 */
#define RVQ_IPC_HANDLE_BYTES 64
RVQ_API int rvq_ipc_export(const void *ptr, void *handle, size_t *offset);
RVQ_API int rvq_ipc_import(const void *handle, size_t offset, void **ptr);
RVQ_API int rvq_ipc_close(void *ptr, size_t offset);

/*
 * Measurement hooks (no counterpart on the pages).
 * rvq_launch_count: number of kernels this library has launched since it was loaded.
 * rvq_profile_enable(1): from now on, bracket every distance-GEMM launch with CUDA events on
 *   its stream (not for use inside stream capture); rvq_profile_enable(0) stops and clears.
 * rvq_profile_read: synchronises on the recorded events and returns the number of RVQ levels the
 *   bracketed launches covered (a per-level distance-GEMM launch counts 1; the all-levels dataflow
 *   encode kernel, which also runs the certificate work, counts L) and their summed device time
 *   in milliseconds since the last enable.
 * rvq_encode_levels_per_launch: for an encode of this shape on the current device, the number of
 *   RVQ levels one bracketed launch covers (L when the all-levels kernel runs, else 1), so that a
 *   profiler can turn rvq_profile_read's totals into per-launch figures.  Same argument checks as
 *   rvq_encode_workspace_size.
 * rvq_encode_candidate_layout: where an encode of this shape keeps its candidate lists in the
 *   workspace, so that a test can read the approximate distances the tensor cores produced:
 *   byte offset `*offset` of an array cand[ceil(N/128)][*slots][128][8] of 8-byte entries
 *   (float d~, int32 id), one list of the 8 lowest d~ = fl(||c||^2) - 2 bf16(r).bf16(c) per
 *   128-row tile, slot and row, written for the LAST level the call encoded (entries with
 *   id < 0 are empty; slots a row tile does not use are left untouched).  Same argument checks
 *   as rvq_encode_workspace_size.
 */
RVQ_API int64_t rvq_launch_count(void);
RVQ_API int rvq_profile_enable(int enable);
RVQ_API int rvq_profile_read(int64_t *gemm_launches, double *gemm_ms);
RVQ_API int rvq_encode_levels_per_launch(int64_t N, int D, int L, int K, int *levels);
RVQ_API int rvq_encode_candidate_layout(int64_t N, int D, int L, int K, size_t *offset, int *slots);

/*
 * Self-test of the bounded waits (no counterpart on the pages).  Every spin of the encode kernels
 * (an mbarrier phase, a grid-wide counter) gives up after a time limit and reports
 * RVQ_ERR_TIMEOUT through the status word instead of hanging the GPU.  This call launches one
 * block that waits on an mbarrier phase nothing completes and on *counter, which the caller keeps
 * at 0, each for at most limit_us microseconds (1 .. 10^7), and then writes RVQ_ERR_TIMEOUT into
 * *status (device int32, first error wins) when both waits gave up as designed, RVQ_ERR_ARG
 * otherwise.  counter and status are caller-owned device pointers.  Returns RVQ_OK when the
 * launch was enqueued, RVQ_ERR_ARG for bad arguments.
 */
RVQ_API int rvq_selftest_wait_timeout(const uint32_t *counter, int32_t *status, int64_t limit_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RVQ_H_ */
