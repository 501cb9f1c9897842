/*
 * kvzip.h -- C ABI of libkvzip: KVzip query-agnostic KV importance scoring,
 * global top-r selection and per-head KV compaction on one NVIDIA B200 (sm_100a).
 *
 * The method (KVzip: Query-Agnostic KV Cache Compression with Context
 * Reconstruction, Kim et al.; blog post sections 4.1-4.5, the scime.ai summary's
 * "Approach" paragraph and the authors' OpenReview rebuttal):
 *
 *   1. Per layer l and KV head h, the reconstruction queries Q_{l,h} in
 *      R^{G x n_in x d} of one chunk attend to the prefilled context keys
 *      K_c in R^{n_c x d} plus the chunk's own causal keys (blog post 4.3.1;
 *      rebuttal: "2x attention FLOPs relative to prefilling").
 *   2. Each context key j is scored by the largest softmax probability any
 *      query row gives it, S_{l,h}[j] = max_{g,i} softmax(Q K^T / sqrt(d))[g,i,j]
 *      (blog post 4.3.2), merged over chunks by a running max (4.5).
 *   3. The top fraction r of all L x H x n_c scores is kept (rebuttal: S has
 *      shape L x H x n_c), which leaves non-uniform per-head budgets (scime.ai
 *      "Measured effects" table), and the kept K/V rows are packed per head
 *      (blog post 4.1, step 5).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers (cudaMalloc / torch CUDA memory)
 *     owned by the caller.  The library never allocates, frees or copies
 *     caller memory, and never synchronises except in kvzip_workspace_status.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it.
 *   - Arguments are validated on the host before anything is enqueued; a
 *     rejected call enqueues nothing and returns KVZIP_ERR_INVALID_ARG (or
 *     KVZIP_ERR_UNSUPPORTED for a valid but unimplemented shape).
 *   - A failed launch returns KVZIP_ERR_CUDA.
 *   - Device pointers must be 16-byte aligned unless stated otherwise.
 *   - Calls that share a workspace must not overlap on the GPU.
 */
#ifndef KVZIP_H_
#define KVZIP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVZIP_OK = 0,
  KVZIP_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, short workspace */
  KVZIP_ERR_UNSUPPORTED = 2,   /* well-formed but not implemented (e.g. head dim 64) */
  KVZIP_ERR_CUDA = 3,          /* a CUDA runtime/driver call or launch failed */
  KVZIP_ERR_TIMEOUT = 4,       /* a kernel gave up waiting on its own pipeline */
  KVZIP_ERR_BOUNDS = 5         /* debug builds: an index failed its bounds check */
} kvzip_status;

typedef enum {
  KVZIP_BF16 = 0,              /* bfloat16 Q / K (tensor-core path) */
  KVZIP_F32 = 1                /* float32 Q / K (CUDA-core path) */
} kvzip_dtype;

/* ------------------------------------------------------------------ scoring */

/* Bytes of workspace kvzip_score_chunk needs for B units of G*n_in query rows:
 * a 256-byte status header plus one float per query row, rows padded to 768. */
size_t kvzip_score_workspace_size(int B, int G, int n_in);

/*
 * Score one reconstruction chunk for B (layer, head) units and merge it into
 * `scores` by a running maximum (blog post 4.3.1, 4.3.2, 4.5).
 *
 *   q       [B][G][n_in][d]  dtype `dt`; query row rho = g*n_in + i, i.e. the
 *                            i-th token of the chunk (repeat-prompt tokens first,
 *                            then the chunk's context tokens) for query head g.
 *   k_ctx   [B][n_c][d]      dtype `dt`; the prefilled context keys K_c.
 *   k_self  [B][n_in][d]     dtype `dt`; the chunk's own keys; row i sees self
 *                            keys 0..i (causal, diagonal included).
 *   scores  [B][n_c] float32, read-modify-write:
 *             scores[b][j] = max(scores[b][j], max_rho P[b][rho][j]) where
 *             P[b][rho][:] = softmax over (n_c context logits, i+1 self logits)
 *             of scale * q . k.  Zero it before the first chunk; 4-byte aligned.
 *             Results lie in [0, 1]: the method's probabilities are > 0, but
 *             the fp32 exponential flushes values below 2^-126 (the smallest
 *             normal float) to 0, so a key whose best probability is below
 *             that scores 0 (and is evicted first).
 *   scale   <= 0 or NaN selects 1/sqrt(d).
 *   d       128 or 256.
 *   workspace / ws_bytes: >= kvzip_score_workspace_size(B, G, n_in) bytes,
 *           256-byte aligned; its first 256 bytes are a sticky status word
 *           that must be zeroed before first use (cudaMemsetAsync) and is read
 *           and cleared by kvzip_workspace_status.
 *
 * B, G, n_in or n_c equal to 0 is a no-op.  Chunks may be scored in any order
 * and re-scoring a chunk leaves `scores` unchanged (max is idempotent), so a
 * caller can checkpoint `scores` between chunks.
 */
kvzip_status kvzip_score_chunk(kvzip_dtype dt, const void* q, const void* k_ctx,
                               const void* k_self, float* scores, int B, int G,
                               int n_in, int n_c, int d, float scale, void* workspace,
                               size_t ws_bytes, void* stream);

/* The two halves of kvzip_score_chunk, same arguments, for callers that time
 * or schedule them separately.  kvzip_score_lse writes each query row's
 * log-sum-exp over its context and visible self keys into the workspace
 * (`scores` is not touched); kvzip_score_colmax then reads them and merges the
 * chunk's per-key maxima into `scores`.  kvzip_score_chunk == lse, then
 * colmax, on the same workspace and stream. */
kvzip_status kvzip_score_lse(kvzip_dtype dt, const void* q, const void* k_ctx,
                             const void* k_self, float* scores, int B, int G, int n_in,
                             int n_c, int d, float scale, void* workspace, size_t ws_bytes,
                             void* stream);
kvzip_status kvzip_score_colmax(kvzip_dtype dt, const void* q, const void* k_ctx,
                                const void* k_self, float* scores, int B, int G, int n_in,
                                int n_c, int d, float scale, void* workspace, size_t ws_bytes,
                                void* stream);

/*
 * kvzip_score_colmax that also counts every score it leaves in `scores` in
 * the selection's first radix round: score_hist[b] += the number of those
 * scores whose |s| bits, shifted right by 19 (the top 13 bits), equal b.
 * Called for a context's last chunk, score_hist is then the round-1
 * histogram of the final scores, and kvzip_select_hist skips its own first
 * read of them.  score_hist: KVZIP_SCORE_HIST_BINS uint32 on the device,
 * zeroed by the caller before the call; other arguments as kvzip_score_colmax.
 * The pages have no counterpart: it fuses work of the selection into the
 * kernel that writes the scores.
 */
#define KVZIP_SCORE_HIST_BINS 8192
kvzip_status kvzip_score_colmax_hist(kvzip_dtype dt, const void* q, const void* k_ctx,
                                     const void* k_self, float* scores, int B, int G, int n_in,
                                     int n_c, int d, float scale, unsigned int* score_hist,
                                     void* workspace, size_t ws_bytes, void* stream);

/*
 * Multi-chunk scoring: all reconstruction chunks of one context in one call
 * (blog post section 4.5: the context is reconstructed chunk by chunk and
 * the chunk scores are merged by a running maximum).  Equivalent to
 * kvzip_score_chunk for chunk 0, 1, ..., n_chunks-1 in order on one stream
 * and workspace; each chunk is two kernel launches (row normalisers, then
 * column maxima).
 *
 *   q, k_self, n_in  HOST arrays of n_chunks entries: device pointers to chunk
 *                    c's queries [B][G][n_in[c]][d] and self keys
 *                    [B][n_in[c]][d], and its row count n_in[c] > 0.  The call
 *                    does not keep the arrays.
 *   workspace        >= kvzip_score_context_workspace_size(B, G, max n_in[c])
 *                    bytes, as for kvzip_score_chunk.
 *
 * Other arguments as for kvzip_score_chunk.  n_chunks = 0 is a no-op.  On an
 * error the chunks before the failing one have been enqueued.
 */
size_t kvzip_score_context_workspace_size(int B, int G, int max_n_in);
kvzip_status kvzip_score_context(kvzip_dtype dt, int n_chunks, const void* const* q,
                                 const void* const* k_self, const int* n_in, const void* k_ctx,
                                 float* scores, int B, int G, int n_c, int d, float scale,
                                 void* workspace, size_t ws_bytes, void* stream);

/* Where kvzip_score_lse (and the first half of kvzip_score_chunk) leaves the
 * row normalisers in the workspace, for callers that read them: the float32 of
 * unit b, query row rho = g*n_in + i, sits at byte
 *     *offset_bytes + 4 * (b * *row_stride + rho)
 * and holds the base-2 log-sum-exp of the row's scaled logits,
 *     log2( sum over its n_c context and i+1 visible self keys of
 *           2^(scale * log2(e) * q . k) ),
 * i.e. the natural-log normaliser times log2(e).  Rows rho >= G*n_in up to
 * the stride are padding.  Valid after the launch completes; the next scoring
 * call on the same workspace overwrites it.  Host-only, no CUDA call. */
kvzip_status kvzip_score_lse_layout(int G, int n_in, size_t* offset_bytes, int64_t* row_stride);

/* Synchronise `stream`, then report (and clear) the status word the kernels
 * leave in `workspace`: KVZIP_OK; KVZIP_ERR_TIMEOUT when a kernel abandoned a
 * pipeline or grid wait (its results for that call are then incomplete); or
 * KVZIP_ERR_INVALID_ARG when kvzip_select_hist found that its histogram does
 * not match the scores. */
kvzip_status kvzip_workspace_status(void* workspace, void* stream);

/* Longest a scoring kernel waits on one pipeline stage before it gives up,
 * records KVZIP_ERR_TIMEOUT in its workspace and returns (default 2 s).
 * Applies to launches enqueued after the call; process-wide.  0 restores the
 * default.  Intended for tests of the timeout path. */
void kvzip_set_wait_timeout_ns(uint64_t ns);

/* Test hook for the timeout path: while on (nonzero), the bf16 scoring
 * kernels' loader warp issues no copies, and the first block of kvzip_select's
 * kernel returns before its first grid barrier, so the waits in them run out
 * after the wait timeout and the call reports KVZIP_ERR_TIMEOUT through
 * kvzip_workspace_status (on the scoring or selection workspace).  Nothing
 * faults or hangs.  Process-wide; applies to launches enqueued after the call.
 * Leave off in normal use. */
void kvzip_set_test_stall(int on);

/* ---------------------------------------------------------------- selection */

/* k = ceil(r * N), the product taken in IEEE double; -1 if r is outside
 * [0, 1] or N < 0.  r is the KEPT fraction ("30% cache ratio"). */
int64_t kvzip_keep_count(double r, int64_t N);

/* Bytes of workspace kvzip_select needs: about 8 * N bytes (a candidate
 * buffer of (flat index, score bits) pairs) plus ~40 KB, 2 KB per 2048 scores
 * up to 2 MB (per-block histograms) and 4 bytes per head. */
size_t kvzip_select_workspace_size(int64_t N, int64_t n_heads);

/*
 * Keep the k largest of the N = n_heads * n_c scores (flat index
 * f = head * n_c + j, head = l*H + h), globally across heads, so per-head
 * budgets follow the scores (scime.ai summary, "Measured effects": uniform
 * head budgets hurt).  Among equal scores the lower flat index is kept first,
 * which makes the mask unique.
 *
 *   scores    [N] float32, >= 0, compared by value: -0.0 equals 0.0 and
 *             +inf ranks above every finite score.  Negative or NaN scores
 *             give an unspecified result that still keeps exactly k and stays
 *             in bounds.
 *   k         0..N (use kvzip_keep_count for a ratio).
 *   n_heads   >= 1, N % n_heads == 0.
 *   keep      [N] uint8 out: 1 = kept.  Any alignment.
 *   offsets   [n_heads + 1] int64 out: offsets[h] = kept rows in heads < h;
 *             offsets[n_heads] = k.  8-byte aligned.
 *   threshold float out or NULL: the k-th largest score, as a non-negative
 *             value (+inf if k == 0).
 *   N < 2^31.
 *   workspace >= kvzip_select_workspace_size(N, n_heads) bytes, 256-byte
 *             aligned.  Its first 4 bytes are a sticky status word, as in the
 *             scoring workspace: zero it before first use; kvzip_workspace_status
 *             reads and clears it.
 *
 * One kernel launch (cooperative: its blocks wait on one another at bounded
 * grid barriers; if a wait runs out, the status word records
 * KVZIP_ERR_TIMEOUT and the mask is incomplete).  The scores are read twice.
 */
kvzip_status kvzip_select(const float* scores, int64_t N, int64_t k, int64_t n_heads,
                          uint8_t* keep, int64_t* offsets, float* threshold,
                          void* workspace, size_t ws_bytes, void* stream);

/*
 * kvzip_select given the round-1 histogram of the scores (score_hist, as
 * kvzip_score_colmax_hist leaves it for a context's last chunk): the scores
 * are read once instead of twice.  The kernel checks the histogram against
 * the scores it reads (the counts above and inside the threshold's bin).  If
 * they disagree, nothing is kept: keep is all 0, offsets all 0, threshold
 * +inf, and the status word records it (kvzip_workspace_status returns
 * KVZIP_ERR_INVALID_ARG).  Other arguments as kvzip_select.  The pages have
 * no counterpart.
 */
kvzip_status kvzip_select_hist(const float* scores, int64_t N, int64_t k, int64_t n_heads,
                               const unsigned int* score_hist, uint8_t* keep, int64_t* offsets,
                               float* threshold, void* workspace, size_t ws_bytes,
                               void* stream);

/*
 * kvzip_select without a workspace, for callers that cannot allocate device
 * memory: e.g. a plugin inside a serving engine whose memory pool has already
 * claimed the GPU, or a latency-critical loop where cudaMalloc (which can
 * block and synchronise the device) is not allowed.  The pages have no
 * counterpart to this; it is a deployment convenience.
 *
 * Same arguments and results as kvzip_select, but the selection scratch is a
 * library-owned static device array of 1 MiB on every GPU that loads the
 * library (held until the process exits).  It runs the multi-launch radix
 * selection (eleven small kernels, three when k == 0), whose scratch is
 * about 40 KB plus 8 bytes per 8192 scores of each head, so it fits problems
 * with roughly n_heads * ceil(n_c / 8192) <= 126000 (all LLaMA3.1-8B /
 * Qwen2.5-14B / Gemma3-12B shapes up to 170K tokens); larger ones return
 * KVZIP_ERR_UNSUPPORTED without launching anything.  N must be >= 1.
 *   - The first call on each device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - All calls on a device share the array: calls that overlap on the GPU
 *     (e.g. on unordered streams) race.  The array keeps the last call's
 *     contents; each call re-initialises what must start at zero.
 *   - Allocates nothing (no cudaMalloc / cudaFree, no allocating library call).
 */
kvzip_status kvzip_select_noalloc(const float* scores, int64_t N, int64_t k, int64_t n_heads,
                                  uint8_t* keep, int64_t* offsets, float* threshold,
                                  void* stream);

/* ------------------------------------------------------- sharded selection */

/*
 * The same global selection when one context's heads are split across ranks
 * (one process per GPU, e.g. tensor-parallel serving where every GPU already
 * holds some KV heads of every layer).  The ranking is global over all L x H x
 * n_c scores (rebuttal: S has shape L x H x n_c; scime.ai "Measured effects":
 * non-uniform head budgets need the global ranking), so the ranks exchange
 * small summaries between the steps below; the caller does the exchange with
 * its own collectives.  Rank r holds a contiguous run of heads, ranks in
 * flat-index order (rank 0 the first heads), N_local = n_heads_local * n_c
 * scores each.  The result equals kvzip_select on the concatenated scores:
 * each rank gets the keep mask of its own scores and offsets over its own
 * heads (offsets[n_heads_local] = rows it keeps).
 *
 *   ws = this rank's workspace (kvzip_select_shard_workspace_size bytes,
 *        256-byte aligned); k = the GLOBAL kept count (<= the sum of N_local).
 *
 *   kvzip_select_shard_begin(k, ws)
 *   for round in 0, 1, 2:
 *     kvzip_select_shard_hist(scores, N_local, round, hist, ws)
 *         hist: device int64[kvzip_select_shard_bins(round)] out, this rank's
 *         counts (the call zeroes it first)
 *     caller: hist <- element-wise SUM of hist over all ranks (all-reduce)
 *     kvzip_select_shard_pick(hist, round, threshold, ws)
 *         threshold: device float or NULL, set to the k-th largest score of
 *         the whole context after round 2
 *   kvzip_select_shard_ties(scores, N_local, n_ties, ws)
 *         n_ties: device int64[1] out, this rank's scores equal to the threshold
 *   caller: tie_counts <- n_ties of every rank, indexed by rank (all-gather)
 *   kvzip_select_shard_mask(scores, N_local, n_heads_local, tie_counts, rank,
 *                           keep, offsets, ws)
 *
 * Every rank must run every step, in this order, with the same k.  Scores
 * 4-byte aligned (16-byte alignment is faster), finite and >= 0;
 * 1 <= N_local < 2^31.  All calls are
 * asynchronous on `stream`; the caller orders its collectives after them.
 */
int kvzip_select_shard_bins(int round);   /* 8192, 1024, 512; 0 for other rounds */
size_t kvzip_select_shard_workspace_size(int64_t N_local, int64_t n_heads_local);
kvzip_status kvzip_select_shard_begin(int64_t k, void* workspace, size_t ws_bytes, void* stream);
kvzip_status kvzip_select_shard_hist(const float* scores, int64_t N_local, int round,
                                     int64_t* hist, void* workspace, size_t ws_bytes,
                                     void* stream);
kvzip_status kvzip_select_shard_pick(const int64_t* hist, int round, float* threshold,
                                     void* workspace, size_t ws_bytes, void* stream);
kvzip_status kvzip_select_shard_ties(const float* scores, int64_t N_local, int64_t* n_ties,
                                     void* workspace, size_t ws_bytes, void* stream);
kvzip_status kvzip_select_shard_mask(const float* scores, int64_t N_local, int64_t n_heads_local,
                                     const int64_t* tie_counts, int rank, uint8_t* keep,
                                     int64_t* offsets, void* workspace, size_t ws_bytes,
                                     void* stream);

/* --------------------------------------------------------------- compaction */

/* Bytes of workspace kvzip_compact needs. */
size_t kvzip_compact_workspace_size(int64_t n_heads, int n_c);

/*
 * Pack the kept rows of K and V into per-head variable-length caches (blog
 * post 4.1, step 5; rebuttal's decoding table: cache size scales with the
 * kept ratio).  For each head, kept positions ascending:
 *   k_out[offsets[h] + t] = k[h][j_t], v_out[...] = v[h][j_t], pos_out[...] = j_t.
 *
 *   k, v      [n_heads][n_c][d] bf16 (rows are copied bit-exactly).
 *   keep      [n_heads * n_c] uint8 (nonzero = kept); offsets as from kvzip_select.
 *   k_out, v_out  [offsets[n_heads]][d] bf16 out; both may be NULL only when
 *             offsets[n_heads] == 0 (nothing kept; nothing is written then).
 *   pos_out   [offsets[n_heads]] int32 out, or NULL.  4-byte aligned.
 *   d         128 or 256.
 */
kvzip_status kvzip_compact(const void* k, const void* v, const uint8_t* keep,
                           const int64_t* offsets, int64_t n_heads, int n_c, int d,
                           void* k_out, void* v_out, int32_t* pos_out, void* workspace,
                           size_t ws_bytes, void* stream);

/* -------------------------------------------------------- decode attention */

/* Bytes of workspace kvzip_decode_attention needs.  Like the scoring
 * workspace it starts with a sticky status word (zero it before first use;
 * kvzip_workspace_status reads and clears it). */
size_t kvzip_decode_workspace_size(int64_t n_heads, int G, int d);

/*
 * One decoding step of attention over the compressed cache from kvzip_compact
 * (rebuttal, decoding-efficiency table: decoding attention latency falls with
 * the kept ratio because only kept KV pairs are read).  For every KV head h
 * and each of its G query heads g:
 *   out[h][g] = softmax(scale * K_h q[h][g]) V_h
 * over head h's kept rows K_h = k_packed[offsets[h] : offsets[h+1]] (same for V).
 * A head with no kept rows gives zeros.
 *   q         [n_heads][G][d] bf16, 16-byte aligned.
 *   k_packed, v_packed  [n_rows][d] bf16 each, 16-byte aligned (may be NULL only
 *             if n_rows is 0).  The kernel reads them by TMA tiles bounded by
 *             n_rows, so no read leaves the buffers whatever offsets holds.
 *   n_rows    rows of k_packed and of v_packed, 0 .. 2^31 - 1; at least
 *             offsets[n_heads] (a head whose range is not inside [0, n_rows)
 *             reads nothing and gives zeros).
 *   offsets   [n_heads + 1] int64 (device).
 *   G         1, 2, 4, 5 or 8; d 128 or 256; scale <= 0 selects 1/sqrt(d).
 *   out       [n_heads][G][d] float32.
 */
kvzip_status kvzip_decode_attention(const void* q, const void* k_packed, const void* v_packed,
                                    int64_t n_rows, const int64_t* offsets, int64_t n_heads,
                                    int G, int d, float scale, float* out, void* workspace,
                                    size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ variants */

/*
 * Sum aggregation (the rebuttal's average-aggregation ablation: sum and
 * average give identical eviction priorities; max ranks better):
 *   scores[b][j] += sum over query rows of softmax(...)[rho][j].
 * Same arguments as kvzip_score_chunk without the dtype: bf16 inputs only.
 * Zero `scores` before the first chunk.
 */
kvzip_status kvzip_score_chunk_sum(const void* q, const void* k_ctx, const void* k_self,
                                   float* scores, int B, int G, int n_in, int n_c, int d,
                                   float scale, void* workspace, size_t ws_bytes, void* stream);

/*
 * Token-level scores (blog post section 4.3.3): token_scores[j] = max over the
 * n_heads = L*H heads of scores[h][j].  Select over them with kvzip_select
 * (n_heads = 1) and turn the position mask into a per-head mask with
 * kvzip_expand_keep.  Exact.
 */
kvzip_status kvzip_token_scores(const float* scores, int64_t n_heads, int64_t n_c,
                                float* token_scores, void* stream);

/* keep[h][j] = keep_pos[j] for every head; offsets[h] = h * kept positions,
 * where kept positions = pos_offsets[1] - pos_offsets[0] (as kvzip_select with
 * n_heads = 1 returns them; device memory). */
kvzip_status kvzip_expand_keep(const uint8_t* keep_pos, const int64_t* pos_offsets,
                               int64_t n_heads, int64_t n_c, uint8_t* keep, int64_t* offsets,
                               void* stream);

/* Bytes of workspace kvzip_select_per_head needs: 8 * n_heads * n_c (a
 * candidate buffer of (position, score bits) pairs). */
size_t kvzip_select_per_head_workspace_size(int64_t n_heads, int64_t n_c);

/*
 * Uniform head budgets (scime.ai summary, "Measured effects": worse than the
 * non-uniform budgets a global ranking gives): keep the k_per_head largest
 * scores inside every head, lower position first among equal scores.
 * offsets[h] = h * k_per_head.  0 <= k_per_head <= n_c; scores 16-byte aligned.
 */
kvzip_status kvzip_select_per_head(const float* scores, int64_t n_heads, int64_t n_c,
                                   int64_t k_per_head, uint8_t* keep, int64_t* offsets,
                                   void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ head scores */

/*
 * Head-level importance, head_scores[h] = max_j scores[h][j] over the n_c
 * positions of each of the n_heads = L*H heads (OpenReview rebuttal, answer on
 * how the head-level scores for the DuoAttention comparison were computed:
 * max over the sequence dimension of the L x H x n_c score tensor).  Exact.
 *   scores       [n_heads][n_c] float32, finite and >= 0; 4-byte aligned.
 *   head_scores  [n_heads] float32 out; 4-byte aligned.
 */
kvzip_status kvzip_head_scores(const float* scores, int64_t n_heads, int64_t n_c,
                               float* head_scores, void* stream);

/* Number of kernel launches the most recent accepted call enqueued
 * (process-wide; for tests and launch accounting). */
int kvzip_last_launch_count(void);

/* ------------------------------------------------------------ debug build */

/* 1 if this library was built with the debug bounds checks (libkvzip_debug.so,
 * `python -m attention_score_reduction_b200.build --debug`), else 0.  In that
 * build the kernels that read or write through computed indices (compaction,
 * both selection paths, the scorer's normaliser tiles and score updates, the
 * decode row ranges) test every such index against its buffer first; a failed
 * test skips the access and sets a flag (no trap, no fault).  Normal builds
 * carry no checks, except that decode attention always skips a head whose
 * rows leave its n_rows (the debug build also sets the flag for it). */
int kvzip_debug_checks(void);

/* Synchronise the current device, then report whether any bounds check failed
 * since the previous call (KVZIP_ERR_BOUNDS) or not (KVZIP_OK), and clear the
 * flags.  Always KVZIP_OK in normal builds. */
kvzip_status kvzip_debug_bounds_status(void);

/* Static, human-readable name of a status code. */
const char* kvzip_status_string(kvzip_status s);

#ifdef __cplusplus
}
#endif

#endif /* KVZIP_H_ */
