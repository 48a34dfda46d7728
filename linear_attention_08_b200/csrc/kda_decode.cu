// KDA decode: one recurrent step per (sequence, head), in place on the FP32 state.
//
// "LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557),
// Methods 1
// (FlashKDA): decode performs the recurrent state update directly; it costs
// about 7 D^2 FLOPs and its memory traffic, about 8 D^2 bytes per head per
// token, is the FP32 state read plus write.  This kernel moves exactly that:
// the state goes HBM -> registers -> HBM once, with 128-bit coalesced
// accesses, and the output is fused into the same pass.
//
// With A = Diag(alpha) S_{t-1}:
//   y = A^T k          (what the gated state retrieves for k)
//   z = A^T q
//   u = beta (v - y)   (delta-rule correction)
//   S_t = A + k u^T    == (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T
//   o = S_t^T q = z + (q . k) u
// The column reductions y and z need the whole state column, so each CTA
// holds one head's state in registers between the reduction and the store.
#include "kda_common.cuh"

namespace kda {

template <int DK, int DV, int THREADS, typename TIn>
__global__ void __launch_bounds__(THREADS, 2)
decode_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
              const float *__restrict__ g, const float *__restrict__ beta,
              float *__restrict__ state, TIn *__restrict__ out, int H) {
  constexpr int V4 = DV / 4;                 // float4 columns per state row
  constexpr int RPP = THREADS / V4;          // rows covered per pass
  constexpr int ROWS = DK / RPP;             // rows held per thread
  static_assert(THREADS % V4 == 0 && DK % RPP == 0, "tile mismatch");
  static_assert(V4 <= 32 && 32 % V4 == 0, "a warp must cover whole rows");

  __shared__ float s_ka[DK];                 // alpha * k
  __shared__ float s_qa[DK];                 // alpha * q
  __shared__ float s_alpha[DK];
  __shared__ float s_k[DK];
  __shared__ float s_v[DV];
  __shared__ float s_u[DV];
  __shared__ float4 s_red[2][RPP][V4];       // partial y, z per row group
  __shared__ float s_qk[THREADS / 32];

  const int unit = blockIdx.x;               // (sequence, head) = row of [N*H]
  const int tid = threadIdx.x;
  const int cg = tid % V4;                   // float4 column owned
  const int rg = tid / V4;                   // first row owned; rows rg + i*RPP

  float4 *S4 = reinterpret_cast<float4 *>(state + (size_t)unit * DK * DV);
  // Issue the state loads first: they are the whole cost of this kernel.
  float4 s[ROWS];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) s[i] = __ldcs(&S4[(rg + i * RPP) * V4 + cg]);

  const size_t vec_k = (size_t)unit * DK, vec_v = (size_t)unit * DV;
  float qk_part = 0.f;
  for (int c = tid; c < DK; c += THREADS) {
    const float kc = to_f32(k[vec_k + c]), qc = to_f32(q[vec_k + c]);
    const float a = __expf(g[vec_k + c]);
    s_alpha[c] = a;
    s_k[c] = kc;
    s_ka[c] = a * kc;
    s_qa[c] = a * qc;
    qk_part += qc * kc;
  }
  for (int j = tid; j < DV; j += THREADS) s_v[j] = to_f32(v[vec_v + j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) qk_part += __shfl_xor_sync(0xffffffffu, qk_part, o);
  if ((tid & 31) == 0) s_qk[tid >> 5] = qk_part;
  __syncthreads();

  float4 y = make_float4(0.f, 0.f, 0.f, 0.f), z = y;
#pragma unroll
  for (int i = 0; i < ROWS; ++i) {
    const int r = rg + i * RPP;
    const float ka = s_ka[r], qa = s_qa[r];
    y.x += ka * s[i].x; y.y += ka * s[i].y; y.z += ka * s[i].z; y.w += ka * s[i].w;
    z.x += qa * s[i].x; z.y += qa * s[i].y; z.z += qa * s[i].z; z.w += qa * s[i].w;
  }
  s_red[0][rg][cg] = y;
  s_red[1][rg][cg] = z;
  __syncthreads();

  if (tid < DV) {
    const int c4 = tid >> 2, lane4 = tid & 3;
    float yy = 0.f, zz = 0.f;
#pragma unroll 8
    for (int r = 0; r < RPP; ++r) {
      yy += reinterpret_cast<const float *>(&s_red[0][r][c4])[lane4];
      zz += reinterpret_cast<const float *>(&s_red[1][r][c4])[lane4];
    }
    float qk = 0.f;
#pragma unroll
    for (int w = 0; w < THREADS / 32; ++w) qk += s_qk[w];
    const float u = beta[unit] * (s_v[tid] - yy);
    s_u[tid] = u;
    out[vec_v + tid] = from_f32<TIn>(zz + qk * u);
  }
  __syncthreads();

  const float4 u4 = reinterpret_cast<const float4 *>(s_u)[cg];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) {
    const int r = rg + i * RPP;
    const float a = s_alpha[r], kc = s_k[r];
    float4 n;
    n.x = a * s[i].x + kc * u4.x;
    n.y = a * s[i].y + kc * u4.y;
    n.z = a * s[i].z + kc * u4.z;
    n.w = a * s[i].w + kc * u4.w;
    __stcs(&S4[r * V4 + cg], n);
  }
}

template <int DK, int DV, typename TIn>
static cudaError_t launch_decode_t(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float *state, void *out, int64_t units,
                                   int H, cudaStream_t stream) {
  constexpr int THREADS = 256;
  decode_kernel<DK, DV, THREADS, TIn><<<(unsigned)units, THREADS, 0, stream>>>(
      (const TIn *)q, (const TIn *)k, (const TIn *)v, g, beta, state, (TIn *)out, H);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_decode_d(int dk, int dv, const void *q, const void *k, const void *v,
                                   const float *g, const float *beta, float *state, void *out,
                                   int64_t units, int H, cudaStream_t stream) {
#define KDA_DEC(DK_, DV_)                                                                   \
  if (dk == DK_ && dv == DV_)                                                               \
    return launch_decode_t<DK_, DV_, TIn>(q, k, v, g, beta, state, out, units, H, stream);
  KDA_DEC(32, 32) KDA_DEC(32, 64) KDA_DEC(32, 128)
  KDA_DEC(64, 32) KDA_DEC(64, 64) KDA_DEC(64, 128)
  KDA_DEC(128, 32) KDA_DEC(128, 64) KDA_DEC(128, 128)
#undef KDA_DEC
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(int dtype, int dk, int dv, const void *q, const void *k, const void *v,
                          const float *g, const float *beta, float *state, void *out,
                          int64_t units, int H, cudaStream_t stream) {
  if (dtype == KDA_DTYPE_BF16)
    return launch_decode_d<__nv_bfloat16>(dk, dv, q, k, v, g, beta, state, out, units, H, stream);
  return launch_decode_d<float>(dk, dv, q, k, v, g, beta, state, out, units, H, stream);
}

}  // namespace kda
