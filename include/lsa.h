/*
 * lsa.h -- C ABI of the Lookahead Sparse Attention (LSA) indexer hot path on NVIDIA B200.
 *
 * The method (pages: "FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long Context via
 * Lookahead Sparse Attention", hyper.ai summary "Method", and the marsggbo blog review,
 * sections 2.2, 3, 3.1, 3.2 and 4.2):  every tau = 64 decode steps a Memory Indexer projects
 * the trigger token's hidden state into indexer queries, scores every preceding compressed
 * index key with I = sigmoid(sum_h w_h ReLU(q_h . K_s)), fetches the entries with I >= 0.5 in
 * any of its three layers from the CPU cold pool into GPU memory, and, at each decode step of
 * the window, the native Lightning Indexer picks its Top-k entries among the fetched ones.
 *
 * Conventions shared by every entry point
 *   - Pointers are device pointers owned by the caller, except the cold pool, which is
 *     caller-owned page-locked host memory mapped into the device address space
 *     (lsa_pool_alloc, cudaHostAlloc(..., cudaHostAllocMapped) or cudaHostRegister(...,
 *     cudaHostRegisterMapped)).  The library keeps no pointer after a call returns and
 *     allocates no device memory: scratch space is the caller's `workspace`.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream); arguments are validated on the host before anything is launched.
 *   - Ragged batches: `seq_offsets` is a DEVICE array of B+1 int64 prefix offsets; sequence b
 *     owns rows seq_offsets[b] .. seq_offsets[b+1]-1 of every [.][T] array, T = total_S =
 *     seq_offsets[B], which the caller also passes by value.  Entry s of sequence b is row
 *     seq_offsets[b] + s.  Every layer has the same entries (an entry is one compressed
 *     position; the layers are OR-combined per entry).
 *   - Errors: a non-LSA_OK status means nothing was launched (or, for LSA_ERR_CUDA, that a
 *     launch failed); lsa_last_error() gives a message for the calling thread.  Kernels that
 *     meet bad data (an index outside its sequence, a count above capacity, a negative or
 *     NaN key scale, decreasing offsets) skip the access and set a device error word, which
 *     lsa_check_device() reads and clears.  No kernel traps and no kernel waits on another.
 *   - Dtypes: LSA_F32 (IEEE binary32), LSA_BF16 (bfloat16), LSA_FP8_E4M3 (OCP E4M3 with one
 *     fp32 scale per key row: key value = scale * decode(code)).
 */
#ifndef LSA_H
#define LSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *lsa_stream_t; /* same handle as cudaStream_t */

typedef enum {
    LSA_OK = 0,
    LSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned buffer, unmapped pool */
    LSA_ERR_UNSUPPORTED = 2,  /* dtype / shape combination without a kernel */
    LSA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    LSA_ERR_DEVICE_CHECK = 4, /* lsa_check_device: a kernel flagged bad data */
    LSA_ERR_WORKSPACE = 5     /* workspace smaller than the *_workspace_size answer */
} lsa_status;

typedef enum { LSA_F32 = 0, LSA_BF16 = 1, LSA_FP8_E4M3 = 2 } lsa_dtype;

/* Largest Top-k the decode-step selection supports. */
#define LSA_MAX_TOPK 4096

/* Message of the last failing call on this thread ("" if none). Never NULL. */
const char *lsa_last_error(void);

/* Library version string. */
const char *lsa_version(void);

/* Number of kernels this library has launched in this process (all threads, all devices). */
uint64_t lsa_launch_count(void);

/* Synchronise `stream`, read and clear the device error word of the current device.
 * Returns LSA_OK, LSA_ERR_DEVICE_CHECK (message lists the flags) or LSA_ERR_CUDA. */
lsa_status lsa_check_device(lsa_stream_t stream);

/* Self-test of the failure detection: one CTA waits, bounded, on a barrier that nothing completes.
 * The wait gives up after its limit (2 s, the limit of every wait inside the pipelined kernels),
 * sets the device error word (pipeline-wait-timeout, read by lsa_check_device) and the kernel
 * returns; the context stays usable.  status_out: device int32 [2], written with {0, 1} (the wait
 * did not complete; the CTA's abort flag is set).  Asynchronous on `stream`. */
lsa_status lsa_selftest_wait_timeout(int32_t *status_out, lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Stage 1 -- Memory-Indexer projections (blog review section 3.1):
 *     c^Q = h W^DQ,   q = c^Q W^IUQ,   w = h W^w,   for each layer l and sequence b.
 *   h      [L][B][d]            dt       hidden state of the trigger token at each indexer layer
 *   W_dq   [L][r][d]            dt       W^DQ stored transposed: row j holds column j (out x in)
 *   W_iuq  [L][n_h*d_I][r]      dt       W^IUQ stored transposed; output o = head*d_I + e
 *   W_w    [L][n_h][d]          dt       W^w stored transposed
 *   q_out  [L][B][n_h][d_I]     dt       queries, rounded to dt (nearest-even)
 *   w_out  [L][B][n_h]          fp32     head weights
 * c^Q is rounded to dt before the second projection; on return the workspace starts with
 * c^Q [L][B][r] in dt.
 * dt: LSA_F32 or LSA_BF16.  Accumulation is fp32.  Workspace: lsa_project_workspace_size.
 * ---------------------------------------------------------------------------------------- */
size_t lsa_project_workspace_size(int L, int B, int d, int r, int n_h, int d_I, lsa_dtype dt);

lsa_status lsa_project(const void *h, const void *W_dq, const void *W_iuq, const void *W_w,
                       lsa_dtype dt, int L, int B, int d, int r, int n_h, int d_I,
                       void *q_out, float *w_out, void *workspace, size_t workspace_bytes,
                       lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Stages 2-4a -- index score, threshold, OR over layers, compaction (blog review sections
 * 3.1 and 4.2; hyper.ai summary "Method"):
 *     x_{l,b,s} = sum_h w_{l,b,h} ReLU(scale_{l,s} q_{l,b,h} . K_{l,s}),   I = sigmoid(x),
 *     entry s of sequence b is fetched iff I_{l,b,s} >= threshold for some layer l.
 * The decision is taken on the logit, x >= log(threshold / (1 - threshold)) in fp32 (x >= 0 at
 * 0.5, so an exact-zero logit is fetched).
 *   q         [L][B][n_h][d_I]   fp32 when kdt = LSA_F32, else bf16
 *   w         [L][B][n_h]        fp32
 *   K         [L][T][d_I]        kdt
 *   k_scale   [L][T]             fp32, required for LSA_FP8_E4M3 (finite, >= 0), else NULL
 *   threshold                    in (0, 1); the pages use 0.5
 *   scores_out  [L][T] fp32      sigmoid scores I (nullable; costs 4 bytes per entry-layer)
 *   mask_out    [T] uint8        1 if fetched (nullable)
 *   idx_out     [T] int32        segment b: the fetched s in ascending order in the first
 *                                count_out[b] slots; the other slots are left unchanged
 *   count_out   [B] int32        number of fetched entries of each sequence
 * Kernels: tcgen05 tensor-core path for n_h = 64, d_I = 128 with bf16 or E4M3 keys (E4M3 on
 * pairs of CTAs for B <= 1024 unless the environment sets LSA_SCORE_PAIR=0; the same result
 * either way); a SIMT path for other shapes (d_I in {32, 64, 128}, n_h <= 128) and for fp32.
 * Workspace: lsa_score_select_workspace_size.
 * ---------------------------------------------------------------------------------------- */
size_t lsa_score_select_workspace_size(int L, int B, int64_t total_S);

lsa_status lsa_memindex_score_select(const void *q, const float *w, const void *K,
                                     const float *k_scale, lsa_dtype kdt,
                                     const int64_t *seq_offsets, int64_t total_S,
                                     int L, int B, int n_h, int d_I, float threshold,
                                     float *scores_out, uint8_t *mask_out,
                                     int32_t *idx_out, int32_t *count_out,
                                     void *workspace, size_t workspace_bytes, lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Stages 2-4a without a workspace.  The method has no counterpart of this entry point: it is
 * a convenience for callers that cannot allocate device memory at the point where they select,
 * for instance a host that runs with a fixed device-memory budget reserved at start-up, or one
 * whose allocator must not be entered on the decode path, and so cannot supply a workspace.
 *
 * Same arguments, outputs and errors as lsa_memindex_score_select, without workspace and
 * workspace_bytes: the scratch is an array of LSA_STATIC_SCORE_SCRATCH_BYTES bytes of device
 * memory owned by the library (one per device, reserved when the library's device code is
 * loaded).  The call allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - Limit: sizes whose lsa_score_select_workspace_size(L, B, total_S) exceeds
 *     LSA_STATIC_SCORE_SCRATCH_BYTES are rejected with LSA_ERR_WORKSPACE and a message naming
 *     both sizes (8 MiB holds, e.g., L = 3, B = 64 and 16 M entries); nothing is launched.
 *   - Nothing needs to start at zero: every scratch byte a call reads, it writes first.
 *   - The first call on each device does a one-time setup with that device current (it looks
 *     up the scratch's device address); make that first call before any stream capture starts.
 *   - One scratch per device: calls that may overlap on one device (different streams, or
 *     different host threads, without an ordering between them) race on it and give wrong
 *     results.  Order them, e.g. issue them on one stream.
 * ---------------------------------------------------------------------------------------- */
#define LSA_STATIC_SCORE_SCRATCH_BYTES (8u << 20)

lsa_status lsa_memindex_score_select_static(const void *q, const float *w, const void *K,
                                            const float *k_scale, lsa_dtype kdt,
                                            const int64_t *seq_offsets, int64_t total_S,
                                            int L, int B, int n_h, int d_I, float threshold,
                                            float *scores_out, uint8_t *mask_out,
                                            int32_t *idx_out, int32_t *count_out,
                                            lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Stage 4b -- fetch C^MemComp from the CPU cold pool into the GPU hot buffer (hyper.ai
 * summary "Method"; blog review section 3):
 *     hot_kv[off_b + j] = pool[off_b + idx[off_b + j]]      for j < count[b]
 * and, when K_sel is given, the same gather of the keys (and scales) of one layer, the keys
 * the decode-step Lightning Indexer scores:
 *     hot_K[off_b + j] = K_sel[off_b + idx[off_b + j]],  hot_scale likewise.
 *   idx, count            as written by lsa_memindex_score_select (device)
 *   pool                  mapped page-locked HOST memory, [T][row_bytes] (nullable together
 *                         with hot_kv: the rows are skipped)
 *   row_bytes             multiple of 16; pool, hot_kv 16-byte aligned
 *   hot_kv                [T][row_bytes] device (capacity T; slots past count untouched)
 *   K_sel, k_scale_sel    [T][d_I] kdt and [T] fp32 (nullable: K_sel NULL skips the keys;
 *                         k_scale_sel required iff kdt = LSA_FP8_E4M3)
 * At least one of pool and K_sel is given.  A rows-only call (K_sel NULL) is a small launch
 * (128 CTAs of 128 threads, up to 8192 sequences) that the host link keeps busy on its own: it is
 * meant to run on a second stream beside the keys-only call (pool NULL) and the Lightning Top-k,
 * which needs only the keys.
 *   hot_K, hot_scale      [T][d_I] and [T] fp32.  hot_K holds kdt for LSA_F32 / LSA_BF16 keys
 *                         and bf16 for LSA_FP8_E4M3 keys: the E4M3 codes are decoded exactly
 *                         (every E4M3 value is a bf16 value); the scale stays in hot_scale.
 * Out-of-range indices or counts are skipped and flagged in the device error word.
 * ---------------------------------------------------------------------------------------- */
lsa_status lsa_fetch_gather(const int32_t *idx, const int32_t *count,
                            const int64_t *seq_offsets, int64_t total_S, int B,
                            const void *pool, size_t row_bytes, void *hot_kv,
                            const void *K_sel, const float *k_scale_sel, lsa_dtype kdt, int d_I,
                            void *hot_K, float *hot_scale, lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Stage 4b, incremental -- the fetch of one window when the previous window's hot rows are still
 * resident.  The pages fetch from the cold pool once per trigger window (hyper.ai summary, one-line
 * summary and "Method"); an entry that the previous window fetched and this one selects again need
 * not cross the host link a second time.
 *     hot_kv[off_b + j] = pool[off_b + idx[off_b + j]]      for j < count[b]       (as above)
 * where a row whose entry s = idx[off_b + j] is also in the previous window's list of sequence b
 * (prev_idx[poff_b + j'] = s, j' < prev_count[b]) is copied on the device from
 * prev_hot_kv[poff_b + j'], and only the other rows cross the host link.
 *   idx, count, seq_offsets, total_S    this window (as written by lsa_memindex_score_select)
 *   prev_idx, prev_count,               the previous window of the same B sequences, whose
 *   prev_seq_offsets, prev_total_S      entries keep their numbers (sequences may have grown);
 *                                       each prev_idx segment ascending (as the select writes it;
 *                                       otherwise rows are fetched that could have been copied)
 *   prev_hot_kv    [prev_total_S][row_bytes] device: the previous window's rows (read only)
 *   pool, row_bytes                     as lsa_fetch_gather; pool laid out at this window's offsets
 *   hot_kv         [total_S][row_bytes] device, must not overlap prev_hot_kv (double buffer)
 *   host_rows_out  nullable device int32: the number of rows read over the host link
 * Workspace: lsa_fetch_incremental_workspace_size (a slot map, the list of rows to fetch and their
 * count).  At most 8192 sequences.  Three launches: lookup, device copy, host rows (128 CTAs, as the
 * rows-only call of lsa_fetch_gather).  The method has no incremental fetch of its own: it is the
 * first widening of the path beyond one window.
 * ---------------------------------------------------------------------------------------- */
size_t lsa_fetch_incremental_workspace_size(int B, int64_t total_S);

lsa_status lsa_fetch_gather_incremental(const int32_t *idx, const int32_t *count,
                                        const int64_t *seq_offsets, int64_t total_S, int B,
                                        const int32_t *prev_idx, const int32_t *prev_count,
                                        const int64_t *prev_seq_offsets, int64_t prev_total_S,
                                        const void *prev_hot_kv, const void *pool, size_t row_bytes,
                                        void *hot_kv, int32_t *host_rows_out,
                                        void *workspace, size_t workspace_bytes, lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Stage 5 -- native Lightning Indexer Top-k over the fetched entries (blog review sections
 * 2.2 and 3.2):  for decode query i of sequence b and fetched slot j < count[b],
 *     y_{b,i,j} = sum_h w'_{b,i,h} ReLU(hot_scale_j q'_{b,i,h} . hot_K_j)
 * and C^CoreComp_{b,i} = the k slots of largest y, reported as entry indices s = idx[off_b+j],
 * ordered by y descending, ties to the smaller s; when count[b] < k the tail is -1 / -inf.
 *   q_dec      [B][tau][n_h][d_I]   fp32 when kdt = LSA_F32, else bf16
 *   w_dec      [B][tau][n_h]        fp32
 *   hot_K, hot_scale                as written by lsa_fetch_gather (hot_scale iff FP8); kdt is
 *                                   the dtype of the original keys (LSA_FP8_E4M3: hot_K is bf16)
 *   idx, count                      as written by lsa_memindex_score_select
 *   k                               1 .. LSA_MAX_TOPK
 *   topk_idx   [B][tau][k] int32
 *   topk_score [B][tau][k] fp32     (nullable)
 * Kernels: tcgen05 tensor-core scoring for n_h = 64, d_I = 128, tau a multiple of 4 (bf16 or
 * E4M3 keys); a SIMT path otherwise.  Then a bucket select per query (4,096 buckets over the
 * query's score range; a radix search inside a crowded bucket).
 * Workspace: lsa_lightning_topk_workspace_size (work plan and the fp32 scores y).
 * ---------------------------------------------------------------------------------------- */
size_t lsa_lightning_topk_workspace_size(int B, int tau, int64_t total_S, int k);

lsa_status lsa_lightning_topk(const void *q_dec, const float *w_dec, const void *hot_K,
                              const float *hot_scale, lsa_dtype kdt,
                              const int32_t *idx, const int32_t *count,
                              const int64_t *seq_offsets, int64_t total_S,
                              int B, int tau, int n_h, int d_I, int k,
                              int32_t *topk_idx, float *topk_score,
                              void *workspace, size_t workspace_bytes, lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Stage 5 for one decode step -- the decode-time form of the native Lightning Indexer Top-k
 * (blog review sections 2.2 and 3.2): at step i of the window every sequence has one query, and
 * its candidates are the entries fetched at the trigger plus the entries compressed since then
 * (they are in device memory, not in the cold pool; the pages leave their handling open).
 *     y_{b,j} as in lsa_lightning_topk for the fetched slots j < count[b], and
 *     y_{b,count[b]+j} = sum_h w_{b,h} ReLU(win_scale_{b,j} q_{b,h} . win_K_{b,j})   for j < win_count[b]
 * Top-k as in lsa_lightning_topk; a window entry j is reported as entry number S_b + j (entries
 * keep counting after the sequence's S_b), so ties still go to the smaller entry number.
 *   q_step, q_batch_stride    query of each sequence: element (b, h, e) at b*q_batch_stride +
 *                             h*d_I + e (bf16, or fp32 for LSA_F32 keys); a column of
 *                             lsa_lightning_topk's q_dec [B][tau][n_h][d_I] works directly
 *   w_step, w_batch_stride    fp32 head weights, (b, h) at b*w_batch_stride + h
 *   hot_K, hot_scale, kdt, idx, count, seq_offsets, total_S   as lsa_lightning_topk
 *   win_K      [B][W][d_I] device, in the hot-key type (bf16 for LSA_BF16 and LSA_FP8_E4M3
 *              keys, fp32 for LSA_F32); win_scale [B][W] fp32 (nullable: scale 1)
 *   win_count  [B] device int32: window entries visible at this step (0 .. W)
 *   topk_idx [B][k] int32, topk_score [B][k] fp32 (nullable)
 * Workspace: lsa_lightning_topk_step_workspace_size.  The call allocates nothing and launches
 * only kernels, so the tau steps of a window can be recorded once in a CUDA graph and replayed.
 * The method has no separate per-step call: this is the second widening beyond one window.
 * ---------------------------------------------------------------------------------------- */
size_t lsa_lightning_topk_step_workspace_size(int B, int64_t total_S, int n_h, int d_I, int W);

lsa_status lsa_lightning_topk_step(const void *q_step, int64_t q_batch_stride,
                                   const float *w_step, int64_t w_batch_stride,
                                   const void *hot_K, const float *hot_scale, lsa_dtype kdt,
                                   const int32_t *idx, const int32_t *count,
                                   const int64_t *seq_offsets, int64_t total_S,
                                   const void *win_K, const float *win_scale,
                                   const int32_t *win_count, int W,
                                   int B, int n_h, int d_I, int k,
                                   int32_t *topk_idx, float *topk_score,
                                   void *workspace, size_t workspace_bytes, lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Golden labels of one future window, the indexer's training targets (blog review section 4.1;
 * hyper.ai summary, "Dataset"; gist.science summary, section 2.2):
 *   for every token i < tau of the window and CSA layer l < Lc: P = softmax over the sequence's
 *   entries of the raw indexer logits z[i][l][.]; nucleus = the entries taken by probability
 *   descending (ties: smaller entry first) until their mass reaches p; golden_i = entries kept by
 *   at least theta layers; label = union of golden_i over the window.  The pages use p = 0.6,
 *   theta = 3 and the 21 CSA layers.
 *   z            [tau][Lc][T] fp32 device, entry s of sequence b at column seq_offsets[b] + s;
 *                1 <= Lc <= 255 and total_S < 2^31 (else LSA_ERR_INVALID_ARG)
 *   label_out    [T] uint8 device: 1 for a golden entry of the window, else 0
 *   nsize_out    [B][tau][Lc] int32 device (nullable): nucleus sizes
 * Softmax masses and their sums are taken in double.  Workspace:
 * lsa_golden_labels_workspace_size (a bit plane per token and layer, cleared by the call).
 * ---------------------------------------------------------------------------------------- */
size_t lsa_golden_labels_workspace_size(int tau, int Lc, int64_t total_S);

lsa_status lsa_golden_labels(const float *z, const int64_t *seq_offsets, int64_t total_S,
                             int B, int tau, int Lc, double p, int theta,
                             uint8_t *label_out, int32_t *nsize_out,
                             void *workspace, size_t workspace_bytes, lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * One training step of the memory indexer (hyper.ai summary, "Method"; blog review section 3):
 * the indexer is trained alone against frozen keys, only W^DQ, W^IUQ and W^w change, with binary
 * cross-entropy on the lookahead scores or, in the pages' final recipe, a focal loss.
 *   forward   as lsa_project and the index score: x_{l,b,s} = sum_h w_h ReLU(scale_s q_h . K_s),
 *             p = sigmoid(x)
 *   loss      mean over the L * total_S (layer, entry) pairs of
 *             -at (1 - pt)^gamma log(pt),  pt = y ? p : 1 - p,  at = alpha < 0 ? 1 : (y ? alpha : 1 - alpha)
 *             (gamma = 0, alpha < 0 is binary cross-entropy); y = labels[offs_b + s] (the window's
 *             golden set, e.g. from lsa_golden_labels; the same target for the L indexers)
 *   backward  the rounding of c and q to dt is passed straight through; ReLU'(a) = 1[a > 0]
 *   h, W_dq, W_iuq, W_w   as lsa_project (dt: LSA_F32 with LSA_F32 keys, LSA_BF16 with LSA_BF16
 *                         or LSA_FP8_E4M3 keys); K [L][T][d_I] kdt, k_scale [L][T] (FP8 only)
 *   labels    [T] uint8 device (0 / 1)
 *   loss_out  [1] double device; g_Wdq [L][r][d], g_Wiuq [L][n_h*d_I][r], g_Ww [L][n_h][d] fp32
 *             device (overwritten)
 * n_h <= 64, d_I <= 128, B <= 16, d and r multiples of 8.  Workspace:
 * lsa_indexer_train_workspace_size.  The method has no
 * training kernel of its own on these pages: this is the fourth widening beyond one window.
 * ---------------------------------------------------------------------------------------- */
size_t lsa_indexer_train_workspace_size(int L, int B, int64_t total_S, int d, int r, int n_h, int d_I,
                                        lsa_dtype dt);

lsa_status lsa_indexer_train_step(const void *h, const void *W_dq, const void *W_iuq, const void *W_w,
                                  lsa_dtype dt, const void *K, const float *k_scale, lsa_dtype kdt,
                                  const uint8_t *labels, const int64_t *seq_offsets, int64_t total_S,
                                  int L, int B, int d, int r, int n_h, int d_I, float gamma, float alpha,
                                  double *loss_out, float *g_Wdq, float *g_Wiuq, float *g_Ww,
                                  void *workspace, size_t workspace_bytes, lsa_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Cold-pool helpers: page-locked host memory mapped into every device's address space
 * (cudaHostAlloc with the Mapped and Portable flags).  The pointer is valid on the host and,
 * unchanged, in kernels.  lsa_pool_free releases memory from lsa_pool_alloc only.
 * ---------------------------------------------------------------------------------------- */
lsa_status lsa_pool_alloc(size_t bytes, void **ptr);
lsa_status lsa_pool_free(void *ptr);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H */
