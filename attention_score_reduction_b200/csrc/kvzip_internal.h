// Internal declarations shared by the host-side C ABI and the kernel files.
#pragma once
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace kvzip {

// Status bits the kernels OR into the workspace header word.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusHistMismatch = 2u;   // kvzip_select_hist: histogram != scores

// Bytes reserved at the front of the scoring workspace for the status word.
constexpr size_t kScoreWsHeader = 256;

// Query rows of one unit are padded to a multiple of this many in the
// log-sum-exp buffer.  Pass 2 reads whole query tiles of it (128 rows at
// d = 128, 64 at d = 256) and pass 1 pads in steps of its 256-row CTAs; the
// scorer asserts at compile time that this divides by both.
constexpr int kRowPad = 768;

struct ScoreArgs {
  const void* q;
  const void* k_ctx;
  const void* k_self;
  float* scores;
  float* lse2;        // [B][R_pad] base-2 log-sum-exp of the scaled logits
  uint32_t* status;   // sticky status word
  int B, G, n_in, n_c, d;
  int R, R_pad;
  float scale;
  uint64_t timeout_ns;
  int passes;         // bit 0: pass 1 (row log-sum-exp), bit 1: pass 2 (column max)
  int test_stall;     // tensor-core scorer only: loader issues nothing (timeout tests)
  int sum_aggregation = 0;  // pass 2 adds column sums instead of taking maxima
  uint32_t* score_hist = nullptr;  // pass 2 (maxima): each resulting score counted in its
                                   // round-1 bin (kScoreHistBins bins, see score_hist_add)
};

// Tensor-core (tcgen05) scorer for bf16 inputs.  Returns a cudaError_t.
cudaError_t launch_score_tc(const ScoreArgs& a, cudaStream_t s, int* launches);
// CUDA-core scorer for fp32 inputs.
cudaError_t launch_score_simt_f32(const ScoreArgs& a, cudaStream_t s, int* launches);

struct SelectArgs {
  const float* scores;
  int64_t N, k, n_heads, n_c;
  uint8_t* keep;
  int64_t* offsets;
  float* threshold;
  void* ws;
  size_t ws_bytes;
  const uint32_t* hist_in = nullptr;   // round-1 histogram of the scores, or null
};
// One cooperative launch, two reads of the scores (kvzip_select).
size_t select_fused_ws_bytes(int64_t N, int64_t n_heads);
cudaError_t launch_select_fused(const SelectArgs& a, uint64_t timeout_ns, int test_stall,
                                cudaStream_t s, int* launches);
// Multi-launch radix select with a small workspace (kvzip_select_noalloc and the
// sharded selection).
size_t select_multipass_ws_bytes(int64_t N, int64_t n_heads);
// Sharded selection (heads split across ranks; histograms summed by the caller).
int shard_bins(int round);
cudaError_t launch_shard_begin(void* ws, int64_t k, cudaStream_t s, int* launches);
cudaError_t launch_shard_hist(const float* scores, int64_t N, int round, long long* hist,
                              void* ws, cudaStream_t s, int* launches);
cudaError_t launch_shard_pick(const long long* hist, int round, float* threshold, void* ws,
                              cudaStream_t s, int* launches);
cudaError_t launch_shard_ties(const float* scores, int64_t N, long long* n_ties, void* ws,
                              cudaStream_t s, int* launches);
cudaError_t launch_shard_mask(const SelectArgs& a, const long long* tie_counts, int rank,
                              cudaStream_t s, int* launches);
// Uniform head budgets: SelectArgs.k is the budget of every head.
size_t select_per_head_ws_bytes(int64_t n_heads, int64_t n_c);
cudaError_t launch_select_per_head(const SelectArgs& a, cudaStream_t s, int* launches);
cudaError_t launch_select_multipass(const SelectArgs& a, cudaStream_t s, int* launches);
// N = 0: zero offsets, threshold +inf, on the stream.
cudaError_t launch_select_empty(int64_t* offsets, int64_t n_heads, float* threshold,
                                cudaStream_t s, int* launches);

struct CompactArgs {
  const void* k;
  const void* v;
  const uint8_t* keep;
  const int64_t* offsets;
  int64_t n_heads;
  int n_c, d;
  void* k_out;
  void* v_out;
  int32_t* pos_out;
  void* ws;
  size_t ws_bytes;
};
size_t compact_ws_bytes(int64_t n_heads, int n_c);
cudaError_t launch_compact(const CompactArgs& a, cudaStream_t s, int* launches);

// Token-level scores and position-mask expansion.
cudaError_t launch_token_scores(const float* scores, int64_t n_heads, int64_t n_c, float* tok,
                                cudaStream_t s, int* launches);
cudaError_t launch_expand_keep(const uint8_t* keep_pos, const int64_t* pos_off, int64_t n_heads,
                               int64_t n_c, uint8_t* keep, int64_t* offsets, cudaStream_t s,
                               int* launches);

// Head-level scores: out[h] = max_j scores[h][j].
cudaError_t launch_head_scores(const float* scores, int64_t n_heads, int64_t n_c, float* out,
                               cudaStream_t s, int* launches);

struct DecodeArgs {
  const void* q;          // [n_heads][G][d] bf16
  const void* k;          // [total][d] bf16, packed head-major
  const void* v;
  int64_t n_rows;         // rows of k and of v
  const int64_t* offsets; // [n_heads + 1]
  int64_t n_heads;
  int G, d;
  float scale;
  float* out;             // [n_heads][G][d] fp32
  void* ws;               // 256-byte status header, then the split partials
  uint64_t timeout_ns;
};
constexpr size_t kDecodeWsHeader = 256;
int decode_splits(int64_t n_heads);
size_t decode_ml_bytes(int64_t n_heads, int G);
size_t decode_ws_bytes(int64_t n_heads, int G, int d);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, int* launches);

// Records the launch count of an accepted call (read by kvzip_last_launch_count).
void note_launches(int launches);

// Debug bounds checks.  Built with -DKVZIP_DEBUG, the kernels that read or
// write through computed indices test each index against the extent of its
// buffer first; a failed test sets this file's flag word and the access is
// skipped (no trap, no fault), so that kvzip_debug_bounds_status can report it
// after the call.  In normal builds in_bounds() is always true and the tests
// compile away.  Every kernel file includes this header and so has its own
// flag word; bounds_flag_*() read and clear them (host, synchronous).
#ifdef KVZIP_DEBUG
static __device__ unsigned int g_bounds_flag;
__device__ __forceinline__ bool in_bounds(bool ok) {
  if (!ok) atomicOr(&g_bounds_flag, 1u);
  return ok;
}
static inline cudaError_t take_bounds_flag(unsigned int* out) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_bounds_flag, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_bounds_flag, &zero, sizeof(zero));
  *out = v;
  return e;
}
#else
__device__ __forceinline__ bool in_bounds(bool) { return true; }
static inline cudaError_t take_bounds_flag(unsigned int* out) {
  *out = 0;
  return cudaSuccess;
}
#endif
cudaError_t bounds_flag_score(unsigned int* out);
cudaError_t bounds_flag_select(unsigned int* out);
cudaError_t bounds_flag_select_fused(unsigned int* out);
cudaError_t bounds_flag_compact(unsigned int* out);
cudaError_t bounds_flag_decode(unsigned int* out);

// Scores are ranked by the bits of |s|: for s >= 0 the bit order is the value
// order, and -0.0 ranks as 0.0 (its raw bits would rank above every score).
// Every kernel that compares or orders score bits reads them through mag.
__host__ __device__ __forceinline__ uint32_t mag(uint32_t w) { return w & 0x7FFFFFFFu; }

// Round-1 histogram of the selection: bin = the top 13 bits of mag(bits).
constexpr int kScoreHistBins = 8192;
constexpr int kScoreHistShift = 19;

// Count score v in its round-1 bin.  Lanes of the calling warp that are here
// together and share a bin add once (scores cluster in a few hundred bins).
__device__ __forceinline__ void score_hist_add(uint32_t* hist, float v) {
  const uint32_t bin = mag(__float_as_uint(v)) >> kScoreHistShift;
  const uint32_t peers = __match_any_sync(__activemask(), bin);
  if ((threadIdx.x & 31u) == static_cast<uint32_t>(__ffs(peers) - 1))
    atomicAdd(hist + bin, static_cast<uint32_t>(__popc(peers)));
}

}  // namespace kvzip
