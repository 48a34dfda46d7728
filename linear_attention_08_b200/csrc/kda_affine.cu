// Affine state algebra for sequence (context) parallelism.
//
// The recurrence is affine in the state it starts from: over a segment of
// tokens, S_out = A S_in + B, where A (D_k x D_k) is the segment's state with
// v = 0 started from the identity and B its state started from zero.  The
// same holds token by token, so the outputs started from S_in are
// o_t = o_t(B) + S_in^T (A_t^T q_t), and A_t^T q_t is the output of the
// v = 0, identity-start run.  These two kernels apply those maps:
//   rows:  y[r, h, :] (+)= x[r, h, :] M[h]      (x: [rows, H, D_k], M: [H, D_k, D_v])
//   state: S_out[h] = A[h] S_in[h] + B[h]        (A: [H, D_k, D_k], S: [H, D_k, D_v])
// The pages name context parallelism among the KDA optimisations
// ("MoonshotAI/Kimi-K3 딥다이브", section 4-1, after the two tricks) without
// detail; this split of the work is the plainest one the recurrence allows.
#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kAThreads = 256;
constexpr int kRowsPerCta = 64;

// One CTA per (block of 64 rows, head): M[h] in shared memory, thread j < D_v
// owns output column j of its rows.
template <typename TIn>
__global__ void __launch_bounds__(kAThreads) affine_rows_kernel(const TIn *__restrict__ x,
                                                                const float *__restrict__ M,
                                                                TIn *__restrict__ y, int64_t rows,
                                                                int H, int Dk, int Dv, int accumulate) {
  extern __shared__ float sm[];
  float *sM = sm;                    // [Dk][Dv]
  float *sx = sM + Dk * Dv;          // [kRowsPerCta][Dk]
  const int h = blockIdx.y, tid = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.x * kRowsPerCta;
  const int nr = (int)((rows - r0) < kRowsPerCta ? (rows - r0) : kRowsPerCta);
  for (int e = tid; e < Dk * Dv; e += kAThreads) sM[e] = M[(size_t)h * Dk * Dv + e];
  for (int e = tid; e < nr * Dk; e += kAThreads) {
    const int r = e / Dk, c = e - r * Dk;
    sx[e] = to_f32(x[((size_t)(r0 + r) * H + h) * Dk + c]);
  }
  __syncthreads();
  // thread (j, part): column j, rows part, part + parts, ...
  const int parts = kAThreads / Dv, j = tid % Dv, part = tid / Dv;
  for (int r = part; r < nr; r += parts) {
    float acc = 0.f;
    for (int c = 0; c < Dk; ++c) acc = fmaf(sx[r * Dk + c], sM[c * Dv + j], acc);
    const size_t o = ((size_t)(r0 + r) * H + h) * Dv + j;
    if (accumulate) acc += to_f32(y[o]);
    y[o] = from_f32<TIn>(acc);
  }
}

// One CTA per head: S_out = A S_in + B, each thread a strided set of entries.
__global__ void __launch_bounds__(kAThreads) affine_state_kernel(const float *__restrict__ A,
                                                                 const float *S, const float *B,
                                                                 float *S_out, int Dk, int Dv) {
  extern __shared__ float sm[];
  float *sS = sm;                    // [Dk][Dv]
  const int h = blockIdx.x, tid = threadIdx.x;
  const float *Ah = A + (size_t)h * Dk * Dk;
  const size_t off = (size_t)h * Dk * Dv;
  for (int e = tid; e < Dk * Dv; e += kAThreads) sS[e] = S[off + e];
  __syncthreads();
  for (int e = tid; e < Dk * Dv; e += kAThreads) {
    const int c = e / Dv, j = e - c * Dv;
    float acc = B ? B[off + e] : 0.f;
    for (int i = 0; i < Dk; ++i) acc = fmaf(Ah[c * Dk + i], sS[i * Dv + j], acc);
    S_out[off + e] = acc;   // S_out may alias S (read from the shared copy) or B (entry e read above)
  }
}

}  // namespace

cudaError_t launch_affine_rows(int dtype, const void *x, const float *M, void *y, int64_t rows,
                               int H, int Dk, int Dv, int accumulate, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)Dk * Dv + (size_t)kRowsPerCta * Dk);
  dim3 grid((unsigned)((rows + kRowsPerCta - 1) / kRowsPerCta), (unsigned)H);
  if (dtype == KDA_DTYPE_BF16) {
    cudaError_t e = cudaFuncSetAttribute(affine_rows_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    affine_rows_kernel<__nv_bfloat16><<<grid, kAThreads, smem, stream>>>(
        (const __nv_bfloat16 *)x, M, (__nv_bfloat16 *)y, rows, H, Dk, Dv, accumulate);
  } else {
    cudaError_t e = cudaFuncSetAttribute(affine_rows_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    affine_rows_kernel<float><<<grid, kAThreads, smem, stream>>>((const float *)x, M, (float *)y,
                                                                 rows, H, Dk, Dv, accumulate);
  }
  return cudaGetLastError();
}

cudaError_t launch_affine_state(const float *A, const float *S, const float *B, float *S_out, int H,
                                int Dk, int Dv, cudaStream_t stream) {
  const size_t smem = sizeof(float) * (size_t)Dk * Dv;
  cudaError_t e = cudaFuncSetAttribute(affine_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  affine_state_kernel<<<(unsigned)H, kAThreads, smem, stream>>>(A, S, B, S_out, Dk, Dv);
  return cudaGetLastError();
}

}  // namespace kda
