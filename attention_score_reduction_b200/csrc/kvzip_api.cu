// Host side of the libkvzip C ABI (declared in include/kvzip.h): argument
// validation, workspace carving and kernel launches.  No allocation, no
// synchronisation (except kvzip_workspace_status), no CPU compute path.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>

#include "kvzip.h"
#include "kvzip_internal.h"

namespace {

std::atomic<uint64_t> g_timeout_ns{2000000000ull};
std::atomic<int> g_last_launches{0};
std::atomic<int> g_test_stall{0};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t row_pad(int64_t R) { return (R + kvzip::kRowPad - 1) / kvzip::kRowPad * kvzip::kRowPad; }

kvzip_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVZIP_OK : KVZIP_ERR_CUDA; }

}  // namespace

void kvzip::note_launches(int launches) { g_last_launches.store(launches); }

extern "C" {

const char* kvzip_status_string(kvzip_status s) {
  switch (s) {
    case KVZIP_OK: return "ok";
    case KVZIP_ERR_INVALID_ARG: return "invalid argument";
    case KVZIP_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case KVZIP_ERR_CUDA: return "CUDA error";
    case KVZIP_ERR_TIMEOUT: return "kernel pipeline wait timed out";
    case KVZIP_ERR_BOUNDS: return "debug bounds check failed";
  }
  return "unknown status";
}

void kvzip_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns == 0 ? 2000000000ull : ns);
}

void kvzip_set_test_stall(int on) { g_test_stall.store(on ? 1 : 0); }

int kvzip_debug_checks(void) {
#ifdef KVZIP_DEBUG
  return 1;
#else
  return 0;
#endif
}

kvzip_status kvzip_debug_bounds_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return KVZIP_ERR_CUDA;
  unsigned int any = 0;
  cudaError_t (*const files[])(unsigned int*) = {
      kvzip::bounds_flag_score, kvzip::bounds_flag_select, kvzip::bounds_flag_select_fused,
      kvzip::bounds_flag_compact, kvzip::bounds_flag_decode};
  for (auto take : files) {
    unsigned int f = 0;
    if (take(&f) != cudaSuccess) return KVZIP_ERR_CUDA;
    any |= f;
  }
  return any ? KVZIP_ERR_BOUNDS : KVZIP_OK;
}

/* Number of kernel launches the most recent successful call enqueued (testing aid). */
int kvzip_last_launch_count(void) { return g_last_launches.load(); }

kvzip_status kvzip_score_lse_layout(int G, int n_in, size_t* offset_bytes, int64_t* row_stride) {
  if (G <= 0 || n_in <= 0 || !offset_bytes || !row_stride) return KVZIP_ERR_INVALID_ARG;
  const int64_t R = static_cast<int64_t>(G) * n_in;
  if (R > INT_MAX - kvzip::kRowPad) return KVZIP_ERR_UNSUPPORTED;
  *offset_bytes = kvzip::kScoreWsHeader;
  *row_stride = row_pad(R);
  return KVZIP_OK;
}

size_t kvzip_score_workspace_size(int B, int G, int n_in) {
  if (B < 0 || G < 0 || n_in < 0) return 0;
  const int64_t R = static_cast<int64_t>(G) * n_in;
  return kvzip::kScoreWsHeader + static_cast<size_t>(B) * static_cast<size_t>(row_pad(R)) * 4;
}

static kvzip_status score_passes(int passes, int sum_agg, kvzip_dtype dt, const void* q, const void* k_ctx,
                                 const void* k_self, float* scores, int B, int G, int n_in,
                                 int n_c, int d, float scale, void* workspace, size_t ws_bytes,
                                 void* stream, unsigned int* score_hist = nullptr) {
  if (dt != KVZIP_BF16 && dt != KVZIP_F32) return KVZIP_ERR_INVALID_ARG;
  if (B < 0 || G < 0 || n_in < 0 || n_c < 0) return KVZIP_ERR_INVALID_ARG;
  if (d != 128 && d != 256) return d > 0 ? KVZIP_ERR_UNSUPPORTED : KVZIP_ERR_INVALID_ARG;
  if (B == 0 || G == 0 || n_in == 0 || n_c == 0) return KVZIP_OK;
  if (!q || !k_ctx || !k_self || !scores || !workspace) return KVZIP_ERR_INVALID_ARG;
  const int64_t R = static_cast<int64_t>(G) * n_in;
  if (R > INT_MAX - kvzip::kRowPad || B > 65535) return KVZIP_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k_ctx, 16) || !aligned(k_self, 16) || !aligned(scores, 4) ||
      !aligned(workspace, 256))
    return KVZIP_ERR_INVALID_ARG;
  if (ws_bytes < kvzip_score_workspace_size(B, G, n_in)) return KVZIP_ERR_INVALID_ARG;
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt(static_cast<float>(d));

  kvzip::ScoreArgs a;
  a.q = q;
  a.k_ctx = k_ctx;
  a.k_self = k_self;
  a.scores = scores;
  a.status = static_cast<uint32_t*>(workspace);
  a.lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kvzip::kScoreWsHeader);
  a.B = B;
  a.G = G;
  a.n_in = n_in;
  a.n_c = n_c;
  a.d = d;
  a.R = static_cast<int>(R);
  a.R_pad = static_cast<int>(row_pad(R));
  a.scale = scale;
  a.timeout_ns = g_timeout_ns.load();
  a.passes = passes;
  a.sum_aggregation = sum_agg;
  a.score_hist = score_hist;
  a.test_stall = g_test_stall.load();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e = (dt == KVZIP_BF16) ? kvzip::launch_score_tc(a, s, &launches)
                                     : kvzip::launch_score_simt_f32(a, s, &launches);
  if (e == cudaErrorInvalidValue) return KVZIP_ERR_INVALID_ARG;  // tensor map rejected the layout
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_score_chunk(kvzip_dtype dt, const void* q, const void* k_ctx,
                               const void* k_self, float* scores, int B, int G, int n_in,
                               int n_c, int d, float scale, void* workspace, size_t ws_bytes,
                               void* stream) {
  return score_passes(3, 0, dt, q, k_ctx, k_self, scores, B, G, n_in, n_c, d, scale, workspace,
                      ws_bytes, stream);
}

kvzip_status kvzip_score_lse(kvzip_dtype dt, const void* q, const void* k_ctx,
                             const void* k_self, float* scores, int B, int G, int n_in, int n_c,
                             int d, float scale, void* workspace, size_t ws_bytes, void* stream) {
  return score_passes(1, 0, dt, q, k_ctx, k_self, scores, B, G, n_in, n_c, d, scale, workspace,
                      ws_bytes, stream);
}

kvzip_status kvzip_score_colmax(kvzip_dtype dt, const void* q, const void* k_ctx,
                                const void* k_self, float* scores, int B, int G, int n_in,
                                int n_c, int d, float scale, void* workspace, size_t ws_bytes,
                                void* stream) {
  return score_passes(2, 0, dt, q, k_ctx, k_self, scores, B, G, n_in, n_c, d, scale, workspace,
                      ws_bytes, stream);
}

kvzip_status kvzip_score_colmax_hist(kvzip_dtype dt, const void* q, const void* k_ctx,
                                     const void* k_self, float* scores, int B, int G, int n_in,
                                     int n_c, int d, float scale, unsigned int* score_hist,
                                     void* workspace, size_t ws_bytes, void* stream) {
  if (!score_hist || !aligned(score_hist, 4)) return KVZIP_ERR_INVALID_ARG;
  return score_passes(2, 0, dt, q, k_ctx, k_self, scores, B, G, n_in, n_c, d, scale, workspace,
                      ws_bytes, stream, score_hist);
}

kvzip_status kvzip_score_chunk_sum(const void* q, const void* k_ctx, const void* k_self,
                                   float* scores, int B, int G, int n_in, int n_c, int d,
                                   float scale, void* workspace, size_t ws_bytes, void* stream) {
  return score_passes(3, 1, KVZIP_BF16, q, k_ctx, k_self, scores, B, G, n_in, n_c, d, scale,
                      workspace, ws_bytes, stream);
}

size_t kvzip_score_context_workspace_size(int B, int G, int max_n_in) {
  return kvzip_score_workspace_size(B, G, max_n_in);
}

kvzip_status kvzip_score_context(kvzip_dtype dt, int n_chunks, const void* const* q,
                                 const void* const* k_self, const int* n_in, const void* k_ctx,
                                 float* scores, int B, int G, int n_c, int d, float scale,
                                 void* workspace, size_t ws_bytes, void* stream) {
  if (n_chunks < 0) return KVZIP_ERR_INVALID_ARG;
  if (n_chunks > 0 && (!q || !k_self || !n_in)) return KVZIP_ERR_INVALID_ARG;
  int max_n_in = 0;
  for (int c = 0; c < n_chunks; ++c) {
    if (!q[c] || !k_self[c] || n_in[c] <= 0) return KVZIP_ERR_INVALID_ARG;
    max_n_in = n_in[c] > max_n_in ? n_in[c] : max_n_in;
  }
  if (ws_bytes < kvzip_score_workspace_size(B, G, max_n_in)) return KVZIP_ERR_INVALID_ARG;
  int launches = 0;
  for (int c = 0; c < n_chunks; ++c) {
    const kvzip_status st = score_passes(3, 0, dt, q[c], k_ctx, k_self[c], scores, B, G, n_in[c],
                                         n_c, d, scale, workspace, ws_bytes, stream);
    if (st != KVZIP_OK) return st;
    launches += g_last_launches.load();
  }
  g_last_launches.store(launches);
  return KVZIP_OK;
}

kvzip_status kvzip_workspace_status(void* workspace, void* stream) {
  if (!workspace) return KVZIP_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVZIP_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KVZIP_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpy(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return KVZIP_ERR_CUDA;
  if (word & kvzip::kStatusTimeout) return KVZIP_ERR_TIMEOUT;
  return (word & kvzip::kStatusHistMismatch) ? KVZIP_ERR_INVALID_ARG : KVZIP_OK;
}

int64_t kvzip_keep_count(double r, int64_t N) {
  if (!(r >= 0.0 && r <= 1.0) || N < 0) return -1;
  return static_cast<int64_t>(std::ceil(r * static_cast<double>(N)));
}

size_t kvzip_select_workspace_size(int64_t N, int64_t n_heads) {
  if (N < 0 || n_heads <= 0) return 0;
  return kvzip::select_fused_ws_bytes(N, n_heads);
}

static kvzip_status select_impl(const float* scores, int64_t N, int64_t k, int64_t n_heads,
                                const unsigned int* score_hist, uint8_t* keep, int64_t* offsets,
                                float* threshold, void* workspace, size_t ws_bytes,
                                void* stream) {
  if (N < 0 || n_heads <= 0 || k < 0 || k > N) return KVZIP_ERR_INVALID_ARG;
  if (N % n_heads != 0 || N >= (int64_t{1} << 31) || n_heads > (int64_t{1} << 24))
    return KVZIP_ERR_INVALID_ARG;
  if (!offsets || !workspace || (N > 0 && (!scores || !keep))) return KVZIP_ERR_INVALID_ARG;
  if (!aligned(offsets, 8) || (scores && !aligned(scores, 16)) || !aligned(workspace, 256) ||
      (threshold && !aligned(threshold, 4)))
    return KVZIP_ERR_INVALID_ARG;
  if (ws_bytes < kvzip_select_workspace_size(N, n_heads)) return KVZIP_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (N == 0) {  // no scores: every head keeps nothing (one enqueued kernel, no sync)
    int launches = 0;
    const cudaError_t e = kvzip::launch_select_empty(offsets, n_heads, threshold, s, &launches);
    if (e == cudaSuccess) g_last_launches.store(launches);
    return from_cuda(e);
  }
  kvzip::SelectArgs a;
  a.scores = scores;
  a.N = N;
  a.k = k;
  a.n_heads = n_heads;
  a.n_c = N / n_heads;
  a.keep = keep;
  a.offsets = offsets;
  a.threshold = threshold;
  a.ws = workspace;
  a.ws_bytes = ws_bytes;
  a.hist_in = score_hist;
  int launches = 0;
  cudaError_t e =
      kvzip::launch_select_fused(a, g_timeout_ns.load(), g_test_stall.load(), s, &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_select(const float* scores, int64_t N, int64_t k, int64_t n_heads,
                          uint8_t* keep, int64_t* offsets, float* threshold, void* workspace,
                          size_t ws_bytes, void* stream) {
  return select_impl(scores, N, k, n_heads, nullptr, keep, offsets, threshold, workspace,
                     ws_bytes, stream);
}

kvzip_status kvzip_select_hist(const float* scores, int64_t N, int64_t k, int64_t n_heads,
                               const unsigned int* score_hist, uint8_t* keep, int64_t* offsets,
                               float* threshold, void* workspace, size_t ws_bytes,
                               void* stream) {
  if (!score_hist || !aligned(score_hist, 4)) return KVZIP_ERR_INVALID_ARG;
  return select_impl(scores, N, k, n_heads, score_hist, keep, offsets, threshold, workspace,
                     ws_bytes, stream);
}

int kvzip_select_shard_bins(int round) { return kvzip::shard_bins(round); }

size_t kvzip_select_shard_workspace_size(int64_t N_local, int64_t n_heads_local) {
  if (N_local < 0 || n_heads_local <= 0) return 0;
  return kvzip::select_multipass_ws_bytes(N_local, n_heads_local);
}

static bool shard_args_ok(const float* scores, int64_t N_local, const void* ws, size_t ws_bytes) {
  return N_local > 0 && N_local < (int64_t{1} << 31) && scores && aligned(scores, 4) && ws &&
         aligned(ws, 256) && ws_bytes >= kvzip::select_multipass_ws_bytes(1, 1);
}

kvzip_status kvzip_select_shard_begin(int64_t k, void* workspace, size_t ws_bytes, void* stream) {
  if (k < 0 || !workspace || !aligned(workspace, 256) ||
      ws_bytes < kvzip::select_multipass_ws_bytes(1, 1))
    return KVZIP_ERR_INVALID_ARG;
  int launches = 0;
  const cudaError_t e =
      kvzip::launch_shard_begin(workspace, k, static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_select_shard_hist(const float* scores, int64_t N_local, int round,
                                     int64_t* hist, void* workspace, size_t ws_bytes,
                                     void* stream) {
  if (!shard_args_ok(scores, N_local, workspace, ws_bytes) || round < 0 || round > 2 || !hist ||
      !aligned(hist, 8))
    return KVZIP_ERR_INVALID_ARG;
  int launches = 0;
  const cudaError_t e = kvzip::launch_shard_hist(scores, N_local, round,
                                                 reinterpret_cast<long long*>(hist), workspace,
                                                 static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_select_shard_pick(const int64_t* hist, int round, float* threshold,
                                     void* workspace, size_t ws_bytes, void* stream) {
  if (round < 0 || round > 2 || !hist || !aligned(hist, 8) || !workspace ||
      !aligned(workspace, 256) || ws_bytes < kvzip::select_multipass_ws_bytes(1, 1) ||
      (threshold && !aligned(threshold, 4)))
    return KVZIP_ERR_INVALID_ARG;
  int launches = 0;
  const cudaError_t e = kvzip::launch_shard_pick(reinterpret_cast<const long long*>(hist), round,
                                                 threshold, workspace,
                                                 static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_select_shard_ties(const float* scores, int64_t N_local, int64_t* n_ties,
                                     void* workspace, size_t ws_bytes, void* stream) {
  if (!shard_args_ok(scores, N_local, workspace, ws_bytes) || !n_ties || !aligned(n_ties, 8))
    return KVZIP_ERR_INVALID_ARG;
  int launches = 0;
  const cudaError_t e = kvzip::launch_shard_ties(scores, N_local,
                                                 reinterpret_cast<long long*>(n_ties), workspace,
                                                 static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_select_shard_mask(const float* scores, int64_t N_local, int64_t n_heads_local,
                                     const int64_t* tie_counts, int rank, uint8_t* keep,
                                     int64_t* offsets, void* workspace, size_t ws_bytes,
                                     void* stream) {
  if (!shard_args_ok(scores, N_local, workspace, ws_bytes) || n_heads_local <= 0 ||
      n_heads_local > (int64_t{1} << 24) || N_local % n_heads_local != 0 || rank < 0 ||
      !tie_counts || !aligned(tie_counts, 8) || !keep || !offsets || !aligned(offsets, 8))
    return KVZIP_ERR_INVALID_ARG;
  if (ws_bytes < kvzip::select_multipass_ws_bytes(N_local, n_heads_local))
    return KVZIP_ERR_INVALID_ARG;
  kvzip::SelectArgs a;
  a.scores = scores;
  a.N = N_local;
  a.k = 0;
  a.n_heads = n_heads_local;
  a.n_c = N_local / n_heads_local;
  a.keep = keep;
  a.offsets = offsets;
  a.threshold = nullptr;
  a.ws = workspace;
  a.ws_bytes = ws_bytes;
  int launches = 0;
  const cudaError_t e = kvzip::launch_shard_mask(a, reinterpret_cast<const long long*>(tie_counts),
                                                 rank, static_cast<cudaStream_t>(stream),
                                                 &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

size_t kvzip_compact_workspace_size(int64_t n_heads, int n_c) {
  if (n_heads <= 0 || n_c < 0) return 0;
  return kvzip::compact_ws_bytes(n_heads, n_c);
}

kvzip_status kvzip_compact(const void* k, const void* v, const uint8_t* keep,
                           const int64_t* offsets, int64_t n_heads, int n_c, int d, void* k_out,
                           void* v_out, int32_t* pos_out, void* workspace, size_t ws_bytes,
                           void* stream) {
  if (n_heads <= 0 || n_c < 0 || n_heads > (int64_t{1} << 24)) return KVZIP_ERR_INVALID_ARG;
  if (d != 128 && d != 256) return d > 0 ? KVZIP_ERR_UNSUPPORTED : KVZIP_ERR_INVALID_ARG;
  if (n_c == 0) return KVZIP_OK;
  if (n_heads * static_cast<int64_t>(n_c) >= (int64_t{1} << 31)) return KVZIP_ERR_UNSUPPORTED;
  if (!k || !v || !keep || !offsets || !workspace) return KVZIP_ERR_INVALID_ARG;
  if ((k_out == nullptr) != (v_out == nullptr)) return KVZIP_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_out, 16) || !aligned(v_out, 16) ||
      !aligned(offsets, 8) || !aligned(workspace, 256) || (pos_out && !aligned(pos_out, 4)))
    return KVZIP_ERR_INVALID_ARG;
  if (ws_bytes < kvzip_compact_workspace_size(n_heads, n_c)) return KVZIP_ERR_INVALID_ARG;
  kvzip::CompactArgs a;
  a.k = k;
  a.v = v;
  a.keep = keep;
  a.offsets = offsets;
  a.n_heads = n_heads;
  a.n_c = n_c;
  a.d = d;
  a.k_out = k_out;
  a.v_out = v_out;
  a.pos_out = pos_out;
  a.ws = workspace;
  a.ws_bytes = ws_bytes;
  int launches = 0;
  cudaError_t e = kvzip::launch_compact(a, static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_head_scores(const float* scores, int64_t n_heads, int64_t n_c,
                               float* head_scores, void* stream) {
  if (n_heads <= 0 || n_c <= 0 || n_heads > (int64_t{1} << 24) || n_c >= (int64_t{1} << 31))
    return KVZIP_ERR_INVALID_ARG;
  if (!scores || !head_scores || !aligned(scores, 4) || !aligned(head_scores, 4))
    return KVZIP_ERR_INVALID_ARG;
  int launches = 0;
  cudaError_t e = kvzip::launch_head_scores(scores, n_heads, n_c, head_scores,
                                            static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

size_t kvzip_decode_workspace_size(int64_t n_heads, int G, int d) {
  if (n_heads <= 0 || G <= 0 || d <= 0) return 0;
  return kvzip::decode_ws_bytes(n_heads, G, d);
}

kvzip_status kvzip_decode_attention(const void* q, const void* k_packed, const void* v_packed,
                                    int64_t n_rows, const int64_t* offsets, int64_t n_heads,
                                    int G, int d, float scale, float* out, void* workspace,
                                    size_t ws_bytes, void* stream) {
  if (n_heads <= 0 || n_heads > 65535 || G <= 0) return KVZIP_ERR_INVALID_ARG;
  if (n_rows < 0 || n_rows > INT32_MAX) return KVZIP_ERR_INVALID_ARG;
  if (n_rows > 0 && (k_packed == nullptr || v_packed == nullptr)) return KVZIP_ERR_INVALID_ARG;
  if (d != 128 && d != 256) return d > 0 ? KVZIP_ERR_UNSUPPORTED : KVZIP_ERR_INVALID_ARG;
  if (G != 1 && G != 2 && G != 4 && G != 5 && G != 8) return KVZIP_ERR_UNSUPPORTED;
  if (!q || !offsets || !out || !workspace) return KVZIP_ERR_INVALID_ARG;
  if ((k_packed == nullptr) != (v_packed == nullptr)) return KVZIP_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_packed, 16) || !aligned(v_packed, 16) ||
      !aligned(offsets, 8) || !aligned(out, 4) || !aligned(workspace, 256))
    return KVZIP_ERR_INVALID_ARG;
  if (ws_bytes < kvzip_decode_workspace_size(n_heads, G, d)) return KVZIP_ERR_INVALID_ARG;
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt(static_cast<float>(d));
  kvzip::DecodeArgs a;
  a.q = q;
  a.k = k_packed;
  a.v = v_packed;
  a.n_rows = n_rows;
  a.offsets = offsets;
  a.n_heads = n_heads;
  a.G = G;
  a.d = d;
  a.scale = scale;
  a.out = out;
  a.ws = workspace;
  a.timeout_ns = g_timeout_ns.load();
  int launches = 0;
  cudaError_t e = kvzip::launch_decode(a, static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_token_scores(const float* scores, int64_t n_heads, int64_t n_c,
                                float* token_scores, void* stream) {
  if (n_heads <= 0 || n_c <= 0 || n_heads * n_c >= (int64_t{1} << 31)) return KVZIP_ERR_INVALID_ARG;
  if (!scores || !token_scores || !aligned(scores, 4) || !aligned(token_scores, 4))
    return KVZIP_ERR_INVALID_ARG;
  int launches = 0;
  cudaError_t e = kvzip::launch_token_scores(scores, n_heads, n_c, token_scores,
                                             static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

kvzip_status kvzip_expand_keep(const uint8_t* keep_pos, const int64_t* pos_offsets,
                               int64_t n_heads, int64_t n_c, uint8_t* keep, int64_t* offsets,
                               void* stream) {
  if (n_heads <= 0 || n_c <= 0 || n_heads * n_c >= (int64_t{1} << 31)) return KVZIP_ERR_INVALID_ARG;
  if (!keep_pos || !pos_offsets || !keep || !offsets || !aligned(pos_offsets, 8) ||
      !aligned(offsets, 8))
    return KVZIP_ERR_INVALID_ARG;
  int launches = 0;
  cudaError_t e = kvzip::launch_expand_keep(keep_pos, pos_offsets, n_heads, n_c, keep, offsets,
                                            static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

size_t kvzip_select_per_head_workspace_size(int64_t n_heads, int64_t n_c) {
  if (n_heads <= 0 || n_c < 0) return 0;
  return kvzip::select_per_head_ws_bytes(n_heads, n_c);
}

kvzip_status kvzip_select_per_head(const float* scores, int64_t n_heads, int64_t n_c,
                                   int64_t k_per_head, uint8_t* keep, int64_t* offsets,
                                   void* workspace, size_t ws_bytes, void* stream) {
  if (n_heads <= 0 || n_heads > 65535 || n_c <= 0 || k_per_head < 0 || k_per_head > n_c)
    return KVZIP_ERR_INVALID_ARG;
  if (n_heads * n_c >= (int64_t{1} << 31)) return KVZIP_ERR_INVALID_ARG;
  if (!scores || !keep || !offsets || !workspace) return KVZIP_ERR_INVALID_ARG;
  if (!aligned(scores, 16) || !aligned(offsets, 8) || !aligned(workspace, 256))
    return KVZIP_ERR_INVALID_ARG;
  if (ws_bytes < kvzip_select_per_head_workspace_size(n_heads, n_c)) return KVZIP_ERR_INVALID_ARG;
  kvzip::SelectArgs a;
  a.scores = scores;
  a.N = n_heads * n_c;
  a.k = k_per_head;
  a.n_heads = n_heads;
  a.n_c = n_c;
  a.keep = keep;
  a.offsets = offsets;
  a.threshold = nullptr;
  a.ws = workspace;
  a.ws_bytes = ws_bytes;
  int launches = 0;
  cudaError_t e = kvzip::launch_select_per_head(a, static_cast<cudaStream_t>(stream), &launches);
  if (e == cudaSuccess) g_last_launches.store(launches);
  return from_cuda(e);
}

}  // extern "C"
