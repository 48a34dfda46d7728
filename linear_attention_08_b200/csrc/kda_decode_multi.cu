// KDA multi-token decode: T_new recurrent steps per (sequence, head) with the
// FP32 state held in registers across the draft (speculative-decoding
// verification).  The step is the decode step of "LLM - Semianalysis, Kimi K3
// 아키텍처" (charstring.tistory.com/2557), Methods 1 (FlashKDA), repeated:
//   y = A^T k, z = A^T q with A = Diag(alpha) S_{t-1};  u = beta (v - y);
//   S_t = A + k u^T;  o = z + (q . k) u.
#include "kda_common.cuh"

namespace kda {

// Multi-token decode (speculative-decoding verification): each (sequence,
// head) runs T_new tokens through the recurrence with its state held in
// registers, writes the output of every token, and stores the state reached
// after the first accept_len[n] tokens (all T_new when accept_len is null).
// One HBM round trip of the state serves all T_new tokens.  Tokens are staged
// in shared memory in groups of kMultiGroup with one batched load, and their
// gates are formed for the whole group before the token loop, so each token
// costs two block barriers and no global-memory latency.
constexpr int kMultiGroup = 8;

template <int DK, int DV, int THREADS, typename TIn>
__global__ void __launch_bounds__(THREADS, 2)
decode_multi_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                    const TIn *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, float *__restrict__ state,
                    TIn *__restrict__ out, const int32_t *__restrict__ accept_len, int T_new,
                    int H) {
  constexpr int V4 = DV / 4;
  constexpr int RPP = THREADS / V4;
  constexpr int ROWS = DK / RPP;
  constexpr int G = kMultiGroup;
  static_assert(THREADS % V4 == 0 && DK % RPP == 0, "tile mismatch");

  __shared__ float s_ka[G][DK], s_qa[G][DK], s_alpha[G][DK], s_k[G][DK];
  __shared__ float s_v[G][DV], s_beta[G], s_qk[G];
  __shared__ float s_u[2][DV];
  __shared__ float4 s_red[2][2][RPP][V4];

  const int unit = blockIdx.x, n = unit / H, h = unit % H;
  const int tid = threadIdx.x, cg = tid % V4, rg = tid / V4;
  const int lane = tid & 31, warp = tid >> 5;
  int acc = T_new;
  if (accept_len) {
    acc = accept_len[n];
    acc = acc < 0 ? 0 : (acc > T_new ? T_new : acc);
  }

  float4 *S4 = reinterpret_cast<float4 *>(state + (size_t)unit * DK * DV);
  // the thread's float4 of each row as two pairs, for the paired FP32 units
  float2 sa[ROWS], sb[ROWS];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) {
    const float4 x = __ldcs(&S4[(rg + i * RPP) * V4 + cg]);
    sa[i] = make_float2(x.x, x.y);
    sb[i] = make_float2(x.z, x.w);
  }

  for (int t0 = 0; t0 < T_new; t0 += G) {
    const int cnt = T_new - t0 < G ? T_new - t0 : G;
    // Stage the group: gates and products for every token at once.
    for (int e = tid; e < cnt * DK; e += THREADS) {
      const int j = e / DK, c = e % DK;
      const size_t off = (((size_t)n * T_new + t0 + j) * H + h) * DK + c;
      const float kc = to_f32(k[off]), qc = to_f32(q[off]);
      const float a = __expf(g[off]);
      s_alpha[j][c] = a;
      s_k[j][c] = kc;
      s_ka[j][c] = a * kc;
      s_qa[j][c] = qc;     // q for now; becomes alpha * q below
    }
    for (int e = tid; e < cnt * DV; e += THREADS) {
      const int j = e / DV, c = e % DV;
      s_v[j][c] = to_f32(v[(((size_t)n * T_new + t0 + j) * H + h) * DV + c]);
    }
    if (tid < cnt) s_beta[tid] = beta[((size_t)n * T_new + t0 + tid) * H + h];
    __syncthreads();
    // q . k per token (one warp per token), then q <- alpha * q
    for (int j = warp; j < cnt; j += THREADS / 32) {
      float qk = 0.f;
      for (int c = lane; c < DK; c += 32) qk += s_qa[j][c] * s_k[j][c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, o);
      if (lane == 0) s_qk[j] = qk;
      for (int c = lane; c < DK; c += 32) s_qa[j][c] *= s_alpha[j][c];
    }
    __syncthreads();

    for (int j = 0; j < cnt; ++j) {
      const int t = t0 + j, p = t & 1;   // parity-indexed buffers: no third barrier
      float2 ya = make_float2(0.f, 0.f), yb = ya, za = ya, zb = ya;
#pragma unroll
      for (int i = 0; i < ROWS; ++i) {
        const int r = rg + i * RPP;
        const float2 ka = make_float2(s_ka[j][r], s_ka[j][r]);
        const float2 qa = make_float2(s_qa[j][r], s_qa[j][r]);
        ya = __ffma2_rn(ka, sa[i], ya);
        yb = __ffma2_rn(ka, sb[i], yb);
        za = __ffma2_rn(qa, sa[i], za);
        zb = __ffma2_rn(qa, sb[i], zb);
      }
      s_red[p][0][rg][cg] = make_float4(ya.x, ya.y, yb.x, yb.y);
      s_red[p][1][rg][cg] = make_float4(za.x, za.y, zb.x, zb.y);
      __syncthreads();
      if (tid < DV) {
        const int c4 = tid >> 2, lane4 = tid & 3;
        float yy = 0.f, zz = 0.f;
#pragma unroll 8
        for (int r = 0; r < RPP; ++r) {
          yy += reinterpret_cast<const float *>(&s_red[p][0][r][c4])[lane4];
          zz += reinterpret_cast<const float *>(&s_red[p][1][r][c4])[lane4];
        }
        const float u = s_beta[j] * (s_v[j][tid] - yy);
        s_u[p][tid] = u;
        out[(((size_t)n * T_new + t) * H + h) * DV + tid] = from_f32<TIn>(zz + s_qk[j] * u);
      }
      __syncthreads();
      const float4 u4 = reinterpret_cast<const float4 *>(s_u[p])[cg];
      const float2 ua = make_float2(u4.x, u4.y), ub = make_float2(u4.z, u4.w);
#pragma unroll
      for (int i = 0; i < ROWS; ++i) {
        const int r = rg + i * RPP;
        const float2 a = make_float2(s_alpha[j][r], s_alpha[j][r]);
        const float2 kc = make_float2(s_k[j][r], s_k[j][r]);
        sa[i] = __ffma2_rn(a, sa[i], __fmul2_rn(kc, ua));
        sb[i] = __ffma2_rn(a, sb[i], __fmul2_rn(kc, ub));
      }
      if (t + 1 == acc)
#pragma unroll
        for (int i = 0; i < ROWS; ++i)
          __stcs(&S4[(rg + i * RPP) * V4 + cg], make_float4(sa[i].x, sa[i].y, sb[i].x, sb[i].y));
    }
    __syncthreads();   // the staged group is overwritten by the next one
  }
}

template <int DK, int DV, typename TIn>
static cudaError_t launch_decode_multi_t(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta, float *state,
                                         void *out, const int32_t *accept_len, int T_new,
                                         int64_t units, int H, cudaStream_t stream) {
  constexpr int THREADS = 256;
  decode_multi_kernel<DK, DV, THREADS, TIn><<<(unsigned)units, THREADS, 0, stream>>>(
      (const TIn *)q, (const TIn *)k, (const TIn *)v, g, beta, state, (TIn *)out, accept_len,
      T_new, H);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_decode_multi_d(int dk, int dv, const void *q, const void *k,
                                         const void *v, const float *g, const float *beta,
                                         float *state, void *out, const int32_t *accept_len,
                                         int T_new, int64_t units, int H, cudaStream_t stream) {
#define KDA_DECM(DK_, DV_)                                                                  \
  if (dk == DK_ && dv == DV_)                                                               \
    return launch_decode_multi_t<DK_, DV_, TIn>(q, k, v, g, beta, state, out, accept_len,   \
                                                T_new, units, H, stream);
  KDA_DECM(32, 32) KDA_DECM(32, 64) KDA_DECM(32, 128)
  KDA_DECM(64, 32) KDA_DECM(64, 64) KDA_DECM(64, 128)
  KDA_DECM(128, 32) KDA_DECM(128, 64) KDA_DECM(128, 128)
#undef KDA_DECM
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_multi(int dtype, int dk, int dv, const void *q, const void *k,
                                const void *v, const float *g, const float *beta, float *state,
                                void *out, const int32_t *accept_len, int T_new, int64_t units,
                                int H, cudaStream_t stream) {
  if (dtype == KDA_DTYPE_BF16)
    return launch_decode_multi_d<__nv_bfloat16>(dk, dv, q, k, v, g, beta, state, out,
                                                accept_len, T_new, units, H, stream);
  return launch_decode_multi_d<float>(dk, dv, q, k, v, g, beta, state, out, accept_len, T_new,
                                      units, H, stream);
}

}  // namespace kda
