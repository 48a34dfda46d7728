// kda_prefill_noalloc: the two-pass prefill for callers that cannot allocate
// device memory at call time (an engine that gave all free memory to its own
// pool, or a runtime whose allocator this library cannot reach).  Its
// workspace is a fixed array compiled into the library.
#include <mutex>

#include "kda_common.cuh"

namespace kda {
kda_status record_cuda_error(cudaError_t e);

namespace {

// The workspace: held on every GPU that loads the library until exit.  Each
// call writes every byte it later reads, so nothing needs clearing; calls
// that overlap on the GPU race on it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];

// Device address of the array on the current device, looked up on the first
// call per device (host code sees only a stand-in for the symbol).
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace kda

extern "C" kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v,
                                          const float *g, const float *beta,
                                          const float *init_state, const int32_t *cu_seqlens,
                                          void *out, float *final_state, int64_t ckpt_interval,
                                          float *ckpt_states, const kda_shape *s,
                                          kda_stream_t stream) {
  const int path = kda_prefill_path(s);
  if (path < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (path != 2) return KDA_ERR_UNSUPPORTED;   // only the two-pass path uses a workspace
  // Smallest workspace: one chunk of every (sequence, head) per window.
  size_t need = kda_prefill_workspace_min_bytes(s);
  if (final_state) need -= (size_t)s->num_seqs * s->num_heads * 128 * 128 * 4;
  if (need > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_UNSUPPORTED;
  void *ws = nullptr;
  const cudaError_t e = kda::scratch_address(&ws);
  if (e != cudaSuccess) return kda::record_cuda_error(e);
  return kda_prefill_ws(q, k, v, g, beta, init_state, cu_seqlens, out, final_state, ckpt_interval,
                        ckpt_states, ws, KDA_NOALLOC_SCRATCH_BYTES, s, stream);
}
