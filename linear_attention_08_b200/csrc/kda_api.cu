// C ABI of the KDA library: argument checks, kernel choice and launch.
#include <stdint.h>
#include <stdio.h>

#include <atomic>
#include <mutex>

#include "kda_common.cuh"

namespace kda {
cudaError_t launch_decode(int dtype, int dk, int dv, const void *q, const void *k, const void *v,
                          const float *g, const float *beta, float *state, void *out,
                          int64_t units, int H, cudaStream_t stream);
cudaError_t launch_prefill_simt(int dtype, int dk, int dv, const void *q, const void *k,
                                const void *v, const float *g, const float *beta,
                                const float *init, const int32_t *cu, void *out, float *fin,
                                int64_t interval, float *ck, const int32_t *pos_cu,
                                const int32_t *positions, float *pos_states, int N, int H,
                                cudaStream_t stream);
cudaError_t launch_decode_multi(int dtype, int dk, int dv, const void *q, const void *k,
                                const void *v, const float *g, const float *beta, float *state,
                                void *out, const int32_t *accept_len, int T_new, int64_t units,
                                int H, int32_t *dev_status, cudaStream_t stream);
bool prefill_tc_supported(int dtype, int dk, int dv, int chunk);
cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *init, const int32_t *cu,
                              void *out, float *fin, int64_t interval, float *ck,
                              const int32_t *pos_cu, const int32_t *positions, float *pos_states,
                              int N, int H, int64_t total_tokens, int32_t *dev_status,
                              cudaStream_t stream);

bool prefill_split_supported(int N);
size_t split_packet_bytes();
size_t split_workspace_full(int N, int H, int64_t T, bool have_final);

cudaError_t launch_prefill_split(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *init, const int32_t *cu, void *out,
                                 float *fin, int64_t interval, float *ck, int N, int H, int64_t T,
                                 void *workspace, size_t ws_bytes, int32_t *dev_status,
                                 cudaStream_t stream, int num_sms);

cudaError_t launch_affine_rows(int dtype, const void *x, const float *M, void *y, int64_t rows,
                               int H, int Dk, int Dv, int accumulate, cudaStream_t stream);
cudaError_t launch_affine_state(const float *A, const float *S, const float *B, float *S_out, int H,
                                int Dk, int Dv, cudaStream_t stream);
size_t backward_workspace_bytes(int N, int H, int64_t T, int Dk, int Dv);
cudaError_t launch_backward(int dtype, const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *init, const int32_t *cu,
                            const float *dout, const float *dfin, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *dinit, float *ws, int N, int H, int Dk,
                            int Dv, int64_t T, cudaStream_t stream);

bool backward_tc_supported(int dtype, int dk, int dv, int N);
size_t backward_tc_workspace_bytes(int N, int H, int64_t T);
cudaError_t launch_backward_tc(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *init, const int32_t *cu,
                               const float *dout, const float *dfin, float *dq, float *dk,
                               float *dv, float *dg, float *dbeta, float *dinit, void *workspace,
                               int N, int H, int64_t T, int32_t *dev_status, cudaStream_t stream,
                               int num_sms);

static thread_local int g_last_cuda_error = 0;
// Backward kernel the last kda_backward call on this thread launched (1 chunked
// tensor-core, 0 SIMT; -1 none yet).
static thread_local int g_last_bwd_path = -1;

// For entry points defined in other files of the library.
kda_status record_cuda_error(cudaError_t e) {
  if (e == cudaSuccess) return KDA_OK;
  g_last_cuda_error = (int)e;
  return KDA_ERR_CUDA;
}

// Largest workspace kda_prefill takes from its pool (longer inputs run in
// windows); kda_set_workspace_pool_cap changes it.
static std::atomic<size_t> g_pool_cap{(size_t)8 << 30};
static const int kMaxDevices = 64;
// Prefill kernel the last prefill call on this thread launched (2, 1, 0; -1 none yet).
static thread_local int g_last_path = -1;
static std::mutex g_pool_mu;
static cudaMemPool_t g_pools[kMaxDevices];
static int g_num_sms[kMaxDevices];

static cudaError_t device_pool(int dev, cudaMemPool_t *out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_pool_mu);
  if (!g_pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaError_t e = cudaMemPoolCreate(&g_pools[dev], &props);
    if (e != cudaSuccess) { g_pools[dev] = nullptr; return e; }
    uint64_t keep = UINT64_MAX;   // keep freed blocks for the next call
    cudaMemPoolSetAttribute(g_pools[dev], cudaMemPoolAttrReleaseThreshold, &keep);
  }
  *out = g_pools[dev];
  return cudaSuccess;
}

static int device_sms(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (!g_num_sms[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_num_sms[dev] = v;
  }
  return g_num_sms[dev];
}

// BF16, D_k = D_v = 128: the tensor-core kernels.  They run 64-token chunks
// whatever chunk size the caller names (16 or 64): the result does not depend
// on the grouping of tokens into chunks, and the pages' 16-token tiles are the
// diagonal blocks of the kernels' UT transform.
static bool tc_shape(const kda_shape *s) {
  return prefill_tc_supported(s->qkv_dtype, s->head_dim_k, s->head_dim_v, 64) &&
         (s->chunk == 16 || s->chunk == 64);
}

// Up to 2048 (sequence, head) units the two-pass kernels are faster (34.9 vs
// 31.8 M tokens/s at 128 units on B200, BF16, D = 128, H = 32; equal at
// 2048); from 4096 units the single-pass grid has the parallelism and is 3 %
// faster.
constexpr int64_t kSplitMaxUnits = 2048;

static bool split_path(const kda_shape *s) {
  return tc_shape(s) && prefill_split_supported(s->num_seqs) &&
         (int64_t)s->num_seqs * s->num_heads <= kSplitMaxUnits;
}

// Windows the two-pass prefill (launch_prefill_split) runs with ws_bytes of
// workspace, 0 if it cannot run: the same count as its launcher makes.  The
// host does not know the longest sequence, so windows are counted up to
// ceil(T / 64) chunks; those past the longest sequence launch both passes with
// nothing to do.
static int64_t split_windows(int N, int H, int64_t T, size_t ws_bytes, bool have_final) {
  if (!prefill_split_supported(N) || ws_bytes < 256) return 0;
  const size_t packet = split_packet_bytes();
  size_t avail = ws_bytes - 256;   // at most this much is lost to the 256-byte alignment
  const int64_t max_chunks = (T + 63) / 64;
  const size_t all_packets = (size_t)H * (size_t)((T + (int64_t)63 * N) / 64);
  if (all_packets * packet <= avail) return 1;
  const size_t state_bytes = (size_t)N * H * 128 * 128 * 4;
  if (!have_final) {
    if (avail < state_bytes) return 0;
    avail -= state_bytes;
  }
  const int64_t wc = (int64_t)(avail / ((size_t)N * H * packet));
  if (wc < 1) return 0;
  return max_chunks > 0 ? (max_chunks + wc - 1) / wc : 1;
}

// Whether the windows the two-pass path would run with ws_bytes of workspace
// are worth it.  A window the host cannot rule out (past the longest
// sequence) still costs both launches, about 5 us + 6 ns per (sequence, head)
// unit; with 1024 x 1024 tokens (H = 32) and an 8 GiB workspace that was 5461
// windows, 1050 ms against 29 ms for the single pass.  The path is kept
// unless those windows cost both more than 5 % of the work (at about 35 M
// tokens/s) and more than 1 ms.
static bool split_worthwhile(const kda_shape *s, size_t ws_bytes, bool have_final) {
  const int64_t units = (int64_t)s->num_seqs * s->num_heads;
  const int64_t w = split_windows(s->num_seqs, s->num_heads, s->total_tokens, ws_bytes, have_final);
  if (w < 1) return false;
  const double idle_us = (double)(w - 1) * (5.0 + 0.006 * (double)units);
  const double work_us = (double)s->total_tokens / 35.0;
  return idle_us <= 0.05 * work_us || idle_us <= 1000.0;
}

static size_t split_min_bytes(const kda_shape *s, bool have_final) {
  return (size_t)s->num_seqs * s->num_heads * split_packet_bytes() +
         (have_final ? 0 : (size_t)s->num_seqs * s->num_heads * 128 * 128 * 4) + 256;
}

static kda_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return KDA_OK;
  g_last_cuda_error = (int)e;
  return KDA_ERR_CUDA;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

static size_t elem_size(int dtype) { return dtype == KDA_DTYPE_BF16 ? 2 : 4; }

// Byte ranges [a, a + na) and [b, b + nb) overlap.
static bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Common shape checks; returns KDA_OK or the status to report.
static kda_status check_shape(const kda_shape *s, bool prefill) {
  if (!s) return KDA_ERR_INVALID_ARGUMENT;
  if (s->num_seqs < 1 || s->num_heads < 1 || s->total_tokens < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (s->qkv_dtype != KDA_DTYPE_F32 && s->qkv_dtype != KDA_DTYPE_BF16)
    return KDA_ERR_INVALID_ARGUMENT;
  if (!head_dim_ok(s->head_dim_k) || !head_dim_ok(s->head_dim_v)) return KDA_ERR_UNSUPPORTED;
  if (prefill && s->chunk != 16 && s->chunk != 64) return KDA_ERR_UNSUPPORTED;
  if ((int64_t)s->num_seqs * s->num_heads > INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (s->dev_status && (reinterpret_cast<uintptr_t>(s->dev_status) & 3u))
    return KDA_ERR_INVALID_ARGUMENT;
  return KDA_OK;
}

}  // namespace kda

using namespace kda;

extern "C" {

int kda_version(void) { return 100; }

int kda_last_cuda_error(void) { return g_last_cuda_error; }

const char *kda_status_string(kda_status s) {
  switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported shape";
    case KDA_ERR_CUDA: return "CUDA error";
    case KDA_ERR_TIMEOUT: return "bounded wait timed out on the device";
  }
  return "unknown status";
}

int64_t kda_ckpt_count(const int32_t *host_cu_seqlens, int32_t num_seqs, int64_t ckpt_interval) {
  if (ckpt_interval <= 0) return 0;
  if (!host_cu_seqlens || num_seqs < 0) return -1;
  int64_t n = 0;
  for (int32_t i = 0; i < num_seqs; ++i) {
    const int64_t len = (int64_t)host_cu_seqlens[i + 1] - host_cu_seqlens[i];
    if (len < 0) return -1;
    n += len / ckpt_interval;
  }
  return n;
}

size_t kda_prefill_workspace_bytes(const kda_shape *s) {
  if (check_shape(s, true) != KDA_OK) return (size_t)-1;
  if (!split_path(s)) return 0;
  return split_workspace_full(s->num_seqs, s->num_heads, s->total_tokens, false);
}

size_t kda_prefill_workspace_min_bytes(const kda_shape *s) {
  if (check_shape(s, true) != KDA_OK) return (size_t)-1;
  return split_path(s) ? split_min_bytes(s, false) : 0;
}

kda_status kda_release_workspace_pool(void) {
  std::lock_guard<std::mutex> lock(g_pool_mu);
  for (int d = 0; d < kMaxDevices; ++d)
    if (g_pools[d]) {
      cudaError_t e = cudaMemPoolTrimTo(g_pools[d], 0);
      if (e != cudaSuccess) return cuda_status(e);
    }
  return KDA_OK;
}

int kda_prefill_path(const kda_shape *s) {
  if (check_shape(s, true) != KDA_OK) return -1;
  if (split_path(s)) {   // as kda_prefill would run it, with a workspace from the pool
    size_t want = split_workspace_full(s->num_seqs, s->num_heads, s->total_tokens, false);
    const size_t cap = g_pool_cap.load();
    if (want > cap) want = cap;
    if (want >= split_min_bytes(s, false) && split_worthwhile(s, want, false)) return 2;
  }
  return tc_shape(s) ? 1 : 0;
}

int kda_last_prefill_path(void) { return g_last_path; }

kda_status kda_set_workspace_pool_cap(size_t bytes) {
  g_pool_cap.store(bytes);
  return KDA_OK;
}

// Workspace modes of prefill_impl.
enum { WS_NONE = 0, WS_CALLER = 1, WS_POOL = 2 };

static kda_status prefill_impl(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *init_state,
                               const int32_t *cu_seqlens, void *out, float *final_state,
                               int64_t ckpt_interval, float *ckpt_states, const int32_t *pos_cu,
                               const int32_t *positions, float *pos_states, int ws_mode,
                               void *workspace, size_t ws_bytes, const kda_shape *s,
                               kda_stream_t stream) {
  kda_status st = check_shape(s, true);
  if (st != KDA_OK) return st;
  const int N = s->num_seqs, H = s->num_heads, DK = s->head_dim_k, DV = s->head_dim_v;
  const int64_t T = s->total_tokens;
  if (!cu_seqlens || !aligned16(cu_seqlens)) return KDA_ERR_INVALID_ARGUMENT;
  if (T > INT32_MAX) return KDA_ERR_UNSUPPORTED;  // cu_seqlens are int32
  if (T > 0) {
    const void *ptrs[] = {q, k, v, g, out};
    for (const void *p : ptrs)
      if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
    if (!beta || (reinterpret_cast<uintptr_t>(beta) & 3u)) return KDA_ERR_INVALID_ARGUMENT;
  }
  if (init_state && !aligned16(init_state)) return KDA_ERR_INVALID_ARGUMENT;
  if (final_state && !aligned16(final_state)) return KDA_ERR_INVALID_ARGUMENT;
  if (ckpt_interval < 0 || ckpt_interval % s->chunk != 0) return KDA_ERR_INVALID_ARGUMENT;
  if ((ckpt_interval > 0) != (ckpt_states != nullptr)) return KDA_ERR_INVALID_ARGUMENT;
  if (ckpt_states && !aligned16(ckpt_states)) return KDA_ERR_INVALID_ARGUMENT;
  if ((positions != nullptr) != (pos_cu != nullptr) || (positions != nullptr) != (pos_states != nullptr))
    return KDA_ERR_INVALID_ARGUMENT;
  if (positions && ((reinterpret_cast<uintptr_t>(positions) & 3u) ||
                    (reinterpret_cast<uintptr_t>(pos_cu) & 3u) || !aligned16(pos_states)))
    return KDA_ERR_INVALID_ARGUMENT;
  const size_t es = elem_size(s->qkv_dtype);
  const size_t n_out = (size_t)T * H * DV * es;
  const size_t n_qk = (size_t)T * H * DK * es, n_v = (size_t)T * H * DV * es;
  const size_t n_g = (size_t)T * H * DK * 4, n_b = (size_t)T * H * 4;
  const size_t n_state = (size_t)N * H * DK * DV * 4;
  if (overlaps(out, n_out, q, n_qk) || overlaps(out, n_out, k, n_qk) ||
      overlaps(out, n_out, v, n_v) || overlaps(out, n_out, g, n_g) ||
      overlaps(out, n_out, beta, n_b) || overlaps(out, n_out, init_state, n_state) ||
      overlaps(out, n_out, final_state, n_state))
    return KDA_ERR_INVALID_ARGUMENT;
  if (final_state && init_state && final_state != init_state &&
      overlaps(final_state, n_state, init_state, n_state))
    return KDA_ERR_INVALID_ARGUMENT;  // exact aliasing is fine, partial overlap is not
  if (ws_mode == WS_CALLER && workspace) {
    if (!aligned16(workspace)) return KDA_ERR_INVALID_ARGUMENT;
    if (overlaps(workspace, ws_bytes, out, n_out) || overlaps(workspace, ws_bytes, q, n_qk) ||
        overlaps(workspace, ws_bytes, k, n_qk) || overlaps(workspace, ws_bytes, v, n_v) ||
        overlaps(workspace, ws_bytes, g, n_g) || overlaps(workspace, ws_bytes, beta, n_b) ||
        overlaps(workspace, ws_bytes, init_state, n_state) ||
        overlaps(workspace, ws_bytes, final_state, n_state) ||
        overlaps(workspace, ws_bytes, ckpt_states, ckpt_states ? 16 : 0))
      return KDA_ERR_INVALID_ARGUMENT;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  // The two-pass kernels store checkpoints at 64-token chunk ends: an interval
  // that is not a multiple of 64 (possible with chunk 16) runs the single pass,
  // which cuts its chunks at every checkpoint.
  if (T > 0 && !positions && ws_mode != WS_NONE && split_path(s) && ckpt_interval % 64 == 0) {
    // Two-pass path when a large enough workspace is at hand.
    const size_t need_min = split_min_bytes(s, final_state != nullptr);
    if (ws_mode == WS_CALLER && workspace && ws_bytes >= need_min &&
        split_worthwhile(s, ws_bytes, final_state != nullptr)) {
      g_last_path = 2;
      return cuda_status(launch_prefill_split(q, k, v, g, beta, init_state, cu_seqlens, out,
                                              final_state, ckpt_interval, ckpt_states, N, H, T,
                                              workspace, ws_bytes, s->dev_status, cs,
                                              device_sms(dev)));
    }
    const size_t cap = g_pool_cap.load();
    if (ws_mode == WS_POOL && cap >= need_min) {
      cudaMemPool_t pool;
      size_t want = split_workspace_full(N, H, T, final_state != nullptr);
      if (want > cap) want = cap;
      void *ws = nullptr;
      if (split_worthwhile(s, want, final_state != nullptr) &&
          device_pool(dev, &pool) == cudaSuccess &&
          cudaMallocFromPoolAsync(&ws, want, pool, cs) == cudaSuccess) {
        g_last_path = 2;
        e = launch_prefill_split(q, k, v, g, beta, init_state, cu_seqlens, out, final_state,
                                 ckpt_interval, ckpt_states, N, H, T, ws, want, s->dev_status, cs,
                                 device_sms(dev));
        const cudaError_t f = cudaFreeAsync(ws, cs);
        return cuda_status(e != cudaSuccess ? e : f);
      }
      cudaGetLastError();   // an allocation that failed runs the single pass (see kda_last_prefill_path)
    }
  }
  if (T > 0 && tc_shape(s)) {
    g_last_path = 1;
    e = launch_prefill_tc(q, k, v, g, beta, init_state, cu_seqlens, out, final_state,
                          ckpt_interval, ckpt_states, pos_cu, positions, pos_states, N, H, T,
                          s->dev_status, cs);
  } else {
    g_last_path = 0;
    e = launch_prefill_simt(s->qkv_dtype, DK, DV, q, k, v, g, beta, init_state, cu_seqlens, out,
                            final_state, ckpt_interval, ckpt_states, pos_cu, positions,
                            pos_states, N, H, cs);
  }
  return cuda_status(e);
}

kda_status kda_prefill(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *init_state, const int32_t *cu_seqlens,
                       void *out, float *final_state, int64_t ckpt_interval,
                       float *ckpt_states, const kda_shape *s, kda_stream_t stream) {
  return prefill_impl(q, k, v, g, beta, init_state, cu_seqlens, out, final_state, ckpt_interval,
                      ckpt_states, nullptr, nullptr, nullptr, WS_POOL, nullptr, 0, s, stream);
}

kda_status kda_prefill_ws(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *init_state, const int32_t *cu_seqlens,
                          void *out, float *final_state, int64_t ckpt_interval,
                          float *ckpt_states, void *workspace, size_t workspace_bytes,
                          const kda_shape *s, kda_stream_t stream) {
  return prefill_impl(q, k, v, g, beta, init_state, cu_seqlens, out, final_state, ckpt_interval,
                      ckpt_states, nullptr, nullptr, nullptr, WS_CALLER, workspace,
                      workspace_bytes, s, stream);
}

kda_status kda_prefill_at(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *init_state, const int32_t *cu_seqlens,
                          void *out, float *final_state, int64_t ckpt_interval,
                          float *ckpt_states, const int32_t *pos_cu, const int32_t *positions,
                          float *pos_states, const kda_shape *s, kda_stream_t stream) {
  return prefill_impl(q, k, v, g, beta, init_state, cu_seqlens, out, final_state, ckpt_interval,
                      ckpt_states, pos_cu, positions, pos_states, positions ? WS_NONE : WS_POOL,
                      nullptr, 0, s, stream);
}

kda_status kda_affine_rows(const void *x, const float *M, void *y, int64_t rows, int32_t accumulate,
                           const kda_shape *s, kda_stream_t stream) {
  if (!s || s->num_heads < 1 || rows < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (s->qkv_dtype != KDA_DTYPE_F32 && s->qkv_dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARGUMENT;
  if (!head_dim_ok(s->head_dim_k) || !head_dim_ok(s->head_dim_v)) return KDA_ERR_UNSUPPORTED;
  const int H = s->num_heads, DK = s->head_dim_k, DV = s->head_dim_v;
  if (rows == 0) return KDA_OK;
  const void *ptrs[] = {x, M, y};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
  const size_t es = elem_size(s->qkv_dtype);
  const size_t ny = (size_t)rows * H * DV * es;
  if (overlaps(y, ny, x, (size_t)rows * H * DK * es) || overlaps(y, ny, M, (size_t)H * DK * DV * 4))
    return KDA_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_affine_rows(s->qkv_dtype, x, M, y, rows, H, DK, DV, accumulate != 0,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

kda_status kda_affine_state(const float *A, const float *S_in, const float *B, float *S_out,
                            const kda_shape *s, kda_stream_t stream) {
  if (!s || s->num_heads < 1) return KDA_ERR_INVALID_ARGUMENT;
  if (!head_dim_ok(s->head_dim_k) || !head_dim_ok(s->head_dim_v)) return KDA_ERR_UNSUPPORTED;
  const int H = s->num_heads, DK = s->head_dim_k, DV = s->head_dim_v;
  const void *ptrs[] = {A, S_in, S_out};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
  if (B && !aligned16(B)) return KDA_ERR_INVALID_ARGUMENT;
  const size_t n_s = (size_t)H * DK * DV * 4;
  if (overlaps(S_out, n_s, A, (size_t)H * DK * DK * 4)) return KDA_ERR_INVALID_ARGUMENT;
  // Each CTA reads its own head of S_in and B before writing that head of
  // S_out: exact aliasing is safe, a partial overlap would race across heads.
  if ((S_out != S_in && overlaps(S_out, n_s, S_in, n_s)) || (B && S_out != B && overlaps(S_out, n_s, B, n_s)))
    return KDA_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_affine_state(A, S_in, B, S_out, H, DK, DV,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

size_t kda_backward_workspace_bytes(const kda_shape *s) {
  if (check_shape(s, false) != KDA_OK) return (size_t)-1;
  if (s->total_tokens > 0 && backward_tc_supported(s->qkv_dtype, s->head_dim_k, s->head_dim_v, s->num_seqs))
    return backward_tc_workspace_bytes(s->num_seqs, s->num_heads, s->total_tokens);
  return backward_workspace_bytes(s->num_seqs, s->num_heads, s->total_tokens, s->head_dim_k,
                                  s->head_dim_v);
}

int kda_last_backward_path(void) { return g_last_bwd_path; }

kda_status kda_backward(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *init_state, const int32_t *cu_seqlens,
                        const float *d_out, const float *d_final_state, float *dq, float *dk,
                        float *dv, float *dg, float *dbeta, float *d_init_state, void *workspace,
                        size_t workspace_bytes, const kda_shape *s, kda_stream_t stream) {
  kda_status st = check_shape(s, false);
  if (st != KDA_OK) return st;
  const int N = s->num_seqs, H = s->num_heads, DK = s->head_dim_k, DV = s->head_dim_v;
  const int64_t T = s->total_tokens;
  if (!cu_seqlens || !aligned16(cu_seqlens)) return KDA_ERR_INVALID_ARGUMENT;
  if (T > INT32_MAX) return KDA_ERR_UNSUPPORTED;
  const size_t es = elem_size(s->qkv_dtype);
  const size_t n_qk = (size_t)T * H * DK * es, n_v = (size_t)T * H * DV * es;
  const size_t n_k4 = (size_t)T * H * DK * 4, n_v4 = (size_t)T * H * DV * 4, n_b = (size_t)T * H * 4;
  const size_t n_state = (size_t)N * H * DK * DV * 4;
  bool chunked = false;
  if (T > 0) {
    const void *ptrs[] = {q, k, v, g, beta, d_out, dq, dk, dv, dg, dbeta};
    for (const void *p : ptrs)
      if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
    // The chunked tensor-core backward when its (larger or smaller) workspace
    // is granted, else the SIMT one.
    chunked = backward_tc_supported(s->qkv_dtype, DK, DV, N) && workspace &&
              workspace_bytes >= backward_tc_workspace_bytes(N, H, T);
    const size_t need = backward_workspace_bytes(N, H, T, DK, DV);
    if (!workspace || !aligned16(workspace) || (!chunked && workspace_bytes < need))
      return KDA_ERR_INVALID_ARGUMENT;
  }
  const void *sp[] = {init_state, d_final_state, d_init_state};
  for (const void *p : sp)
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
  // outputs must overlap no input and no other output
  const void *outs[] = {dq, dk, dv, dg, dbeta, d_init_state, workspace};
  const size_t out_n[] = {n_k4, n_k4, n_v4, n_k4, n_b, n_state, workspace_bytes};
  const void *ins[] = {q, k, v, g, beta, init_state, d_out, d_final_state, cu_seqlens};
  const size_t in_n[] = {n_qk, n_qk, n_v, n_k4, n_b, n_state, n_v4, n_state, (size_t)(N + 1) * 4};
  for (int i = 0; i < 7; ++i) {
    for (int j = 0; j < 9; ++j)
      if (overlaps(outs[i], out_n[i], ins[j], in_n[j])) return KDA_ERR_INVALID_ARGUMENT;
    for (int j = i + 1; j < 7; ++j)
      if (overlaps(outs[i], out_n[i], outs[j], out_n[j])) return KDA_ERR_INVALID_ARGUMENT;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (chunked) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    g_last_bwd_path = 1;
    return cuda_status(launch_backward_tc(q, k, v, g, beta, init_state, cu_seqlens, d_out,
                                         d_final_state, dq, dk, dv, dg, dbeta, d_init_state,
                                         workspace, N, H, T, s->dev_status, cs, device_sms(dev)));
  }
  g_last_bwd_path = 0;
  return cuda_status(launch_backward(s->qkv_dtype, q, k, v, g, beta, init_state, cu_seqlens, d_out,
                                     d_final_state, dq, dk, dv, dg, dbeta, d_init_state,
                                     reinterpret_cast<float *>(workspace), N, H, DK, DV, T, cs));
}

kda_status kda_decode(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, float *state_inout, void *out, const kda_shape *s,
                      kda_stream_t stream) {
  kda_status st = check_shape(s, false);
  if (st != KDA_OK) return st;
  if (s->total_tokens != s->num_seqs) return KDA_ERR_INVALID_ARGUMENT;
  const void *ptrs[] = {q, k, v, g, state_inout, out};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
  if (!beta || (reinterpret_cast<uintptr_t>(beta) & 3u)) return KDA_ERR_INVALID_ARGUMENT;
  const int64_t units = (int64_t)s->num_seqs * s->num_heads;
  const size_t es = elem_size(s->qkv_dtype);
  const size_t n_out = (size_t)units * s->head_dim_v * es;
  const size_t n_state = (size_t)units * s->head_dim_k * s->head_dim_v * 4;
  if (overlaps(out, n_out, state_inout, n_state) ||
      overlaps(out, n_out, q, (size_t)units * s->head_dim_k * es) ||
      overlaps(out, n_out, k, (size_t)units * s->head_dim_k * es) ||
      overlaps(out, n_out, v, n_out) || overlaps(out, n_out, g, (size_t)units * s->head_dim_k * 4))
    return KDA_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_decode(s->qkv_dtype, s->head_dim_k, s->head_dim_v, q, k, v, g, beta,
                                   state_inout, out, units, s->num_heads,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

kda_status kda_decode_multi(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float *state_inout, void *out,
                            const int32_t *accept_len, int32_t tokens_per_seq,
                            const kda_shape *s, kda_stream_t stream) {
  kda_status st = check_shape(s, false);
  if (st != KDA_OK) return st;
  if (tokens_per_seq < 1 || tokens_per_seq > 64) return KDA_ERR_INVALID_ARGUMENT;
  if (s->total_tokens != (int64_t)s->num_seqs * tokens_per_seq) return KDA_ERR_INVALID_ARGUMENT;
  const void *ptrs[] = {q, k, v, g, state_inout, out};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
  if (!beta || (reinterpret_cast<uintptr_t>(beta) & 3u)) return KDA_ERR_INVALID_ARGUMENT;
  if (accept_len && (reinterpret_cast<uintptr_t>(accept_len) & 3u)) return KDA_ERR_INVALID_ARGUMENT;
  const int64_t units = (int64_t)s->num_seqs * s->num_heads;
  const int64_t T = s->total_tokens, H = s->num_heads;
  const size_t es = elem_size(s->qkv_dtype);
  const size_t n_out = (size_t)T * H * s->head_dim_v * es;
  const size_t n_state = (size_t)units * s->head_dim_k * s->head_dim_v * 4;
  if (overlaps(out, n_out, state_inout, n_state) ||
      overlaps(out, n_out, q, (size_t)T * H * s->head_dim_k * es) ||
      overlaps(out, n_out, k, (size_t)T * H * s->head_dim_k * es) ||
      overlaps(out, n_out, v, n_out) || overlaps(out, n_out, g, (size_t)T * H * s->head_dim_k * 4))
    return KDA_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_decode_multi(s->qkv_dtype, s->head_dim_k, s->head_dim_v, q, k, v, g,
                                         beta, state_inout, out, accept_len, tokens_per_seq,
                                         units, s->num_heads, s->dev_status,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace kda {
__global__ void selftest_wait_kernel(int32_t *dev_status, int64_t max_polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // Nothing ever arrives: the wait must give up and report.
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, max_polls)) report(dev_status, KDA_ERR_TIMEOUT);
}
}  // namespace kda

extern "C" kda_status kda_selftest_bounded_wait(int32_t *dev_status, int64_t max_polls,
                                                kda_stream_t stream) {
  if (!dev_status || max_polls < 0 || max_polls > (int64_t(1) << 24)) return KDA_ERR_INVALID_ARGUMENT;
  kda::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(dev_status,
                                                                                  max_polls);
  return kda::cuda_status(cudaGetLastError());
}
