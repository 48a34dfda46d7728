// KDA chunked prefill on the SIMT FP32 pipes.
//
// This is the FP32 path: it serves FP32 inputs (where the result must stay
// within 1e-4 of the FP64 definition) and any head size the tensor-core
// kernel does not cover.  It follows the chunked form of the recurrence
// ("LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557), Methods 1: prefill groups tokens into
// chunks, unrolls the recurrence and computes it with matrix products; deep
// dive section 4-1: 16-token tiles, dense work inside a tile and a
// recurrence between tiles).  It always works in 16-token tiles; the result
// does not depend on the tile size, so a requested chunk of 64 runs as four
// tiles here.
//
// For one tile of L <= 16 tokens starting from state S0, with the inclusive
// per-channel cumulative log-decay Gam_r = sum_{s<=r} g_s:
//   M_ri = beta_r sum_c k_rc k_ic exp(Gam_rc - Gam_ic)      (i < r)
//   P_ri = sum_c q_rc k_ic exp(Gam_rc - Gam_ic)             (i <= r)
//   (I + M) U = diag(beta) (V - Kt S0),   Kt_r = k_r exp(Gam_r)
//   O = Qt S0 + P U,                      Qt_r = q_r exp(Gam_r)
//   S = Diag(exp(Gam_L)) S0 + Kh^T U,     Kh_r = k_r exp(Gam_L - Gam_r)
// Tokens past the end of a sequence are identity tokens (q = k = v = 0,
// beta = 0, g = 0), which leave the state unchanged.
//
// One CTA owns one (sequence, head, 32-column slice of D_v): the value
// columns of the recurrence are independent, so slices need no exchange.
#include "kda_common.cuh"

namespace kda {

constexpr int kSimtTile = 16;
constexpr int kSimtSlice = 32;
constexpr int kSimtThreads = 256;

template <int DK>
struct SimtSmem {
  float S[DK][kSimtSlice];
  float q[kSimtTile][DK];
  float k[kSimtTile][DK];
  float gam[kSimtTile][DK];   // g, then the inclusive cumulative sum
  float eg[kSimtTile][DK];    // exp(Gam_r)
  float eh[kSimtTile][DK];    // exp(Gam_L - Gam_r)
  float v[kSimtTile][kSimtSlice];
  float u[kSimtTile][kSimtSlice];
  float M[kSimtTile][kSimtTile + 1];
  float P[kSimtTile][kSimtTile + 1];
  float beta[kSimtTile];
};

template <int DK, typename TIn>
__global__ void __launch_bounds__(kSimtThreads)
prefill_simt_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                    const TIn *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, const float *__restrict__ init_state,
                    const int32_t *__restrict__ cu_seqlens, TIn *__restrict__ out,
                    float *__restrict__ final_state, int64_t ckpt_interval,
                    float *__restrict__ ckpt_states, const int32_t *__restrict__ pos_cu,
                    const int32_t *__restrict__ positions, float *__restrict__ pos_states,
                    int H, int DV) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem<DK> &sm = *reinterpret_cast<SimtSmem<DK> *>(smem_raw);
  constexpr int T = kSimtTile, W = kSimtSlice, NT = kSimtThreads;
  const int unit = blockIdx.x;                 // seq * H + h
  const int seq = unit / H, h = unit % H;
  const int col0 = blockIdx.y * W;             // first value column of this slice
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int64_t t_begin = cu_seqlens[seq], t_end = cu_seqlens[seq + 1], T_seq = t_end - t_begin;
  int64_t ck_slot = 0;
  if (ckpt_interval > 0)
    for (int j = 0; j < seq; ++j) ck_slot += (cu_seqlens[j + 1] - cu_seqlens[j]) / ckpt_interval;
  int pi = positions ? pos_cu[seq] : 0;
  const int pe = positions ? pos_cu[seq + 1] : 0;

  const size_t state_off = (size_t)unit * DK * DV;
  for (int e = tid; e < DK * W; e += NT) {
    const int c = e / W, j = e % W;
    sm.S[c][j] = init_state ? init_state[state_off + (size_t)c * DV + col0 + j] : 0.f;
  }
  // Copy the state slice into a [.., H, DK, DV] array (after a barrier).
  auto store_state = [&](float *base_ptr, int64_t slot) {
    __syncthreads();
    float *dst = base_ptr + ((size_t)slot * H + h) * DK * DV;
    for (int e = tid; e < DK * W; e += NT) {
      const int c = e / W, j = e % W;
      dst[(size_t)c * DV + col0 + j] = sm.S[c][j];
    }
  };
  while (pi < pe && positions[pi] <= 0) store_state(pos_states, pi++);   // initial state

  // Tiles end at the next checkpoint boundary or explicit position, so every
  // stored state is the state at a tile end (tiling does not change the result).
  for (int64_t done = 0; done < T_seq;) {
    const int64_t c0 = t_begin + done;
    int64_t m = T_seq - done < T ? T_seq - done : T;
    if (ckpt_interval > 0) {
      const int64_t to_ck = ckpt_interval - done % ckpt_interval;
      m = to_ck < m ? to_ck : m;
    }
    if (pi < pe) {
      const int64_t to_pos = (int64_t)positions[pi] - done;
      m = to_pos < m ? to_pos : m;
    }
    const int L = (int)m;
    __syncthreads();  // previous tile fully consumed
    for (int e = tid; e < T * DK; e += NT) {
      const int r = e / DK, c = e % DK;
      const size_t off = ((size_t)(c0 + r) * H + h) * DK + c;
      const bool in = r < L;
      sm.q[r][c] = in ? to_f32(q[off]) : 0.f;
      sm.k[r][c] = in ? to_f32(k[off]) : 0.f;
      sm.gam[r][c] = in ? g[off] : 0.f;
    }
    for (int e = tid; e < T * W; e += NT) {
      const int r = e / W, j = e % W;
      sm.v[r][j] = r < L ? to_f32(v[((size_t)(c0 + r) * H + h) * DV + col0 + j]) : 0.f;
    }
    if (tid < T) sm.beta[tid] = tid < L ? beta[(size_t)(c0 + tid) * H + h] : 0.f;
    __syncthreads();

    // Gate prep: inclusive cumulative sum over the tile, per channel.
    for (int c = tid; c < DK; c += NT) {
      float acc = 0.f;
#pragma unroll
      for (int r = 0; r < T; ++r) {
        acc += sm.gam[r][c];
        sm.gam[r][c] = acc;
      }
#pragma unroll
      for (int r = 0; r < T; ++r) {
        sm.eg[r][c] = expf(sm.gam[r][c]);
        sm.eh[r][c] = expf(acc - sm.gam[r][c]);
      }
    }
    __syncthreads();

    // Gated Gram products M and P: one warp per (r, i) pair, lanes over channels.
    for (int p = warp; p < T * T; p += NT / 32) {
      const int r = p / T, i = p % T;
      if (i > r) continue;  // uniform across the warp
      float m = 0.f, pr = 0.f;
#pragma unroll
      for (int c = lane; c < DK; c += 32) {
        const float e = expf(sm.gam[r][c] - sm.gam[i][c]);
        const float ki = sm.k[i][c] * e;
        m += sm.k[r][c] * ki;
        pr += sm.q[r][c] * ki;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        m += __shfl_xor_sync(0xffffffffu, m, o);
        pr += __shfl_xor_sync(0xffffffffu, pr, o);
      }
      if (lane == 0) {
        sm.M[r][i] = i < r ? sm.beta[r] * m : 0.f;
        sm.P[r][i] = pr;
      }
    }
    // Right-hand side diag(beta)(V - Kt S0).
    for (int e = tid; e < T * W; e += NT) {
      const int r = e / W, j = e % W;
      float w = 0.f;
#pragma unroll 8
      for (int c = 0; c < DK; ++c) w += sm.k[r][c] * sm.eg[r][c] * sm.S[c][j];
      sm.u[r][j] = sm.beta[r] * (sm.v[r][j] - w);
    }
    __syncthreads();

    // Unit lower-triangular solve (I + M) U = rhs, one column per thread.
    if (tid < W) {
      const int j = tid;
      float ucol[T];
#pragma unroll
      for (int r = 0; r < T; ++r) {
        float x = sm.u[r][j];
#pragma unroll
        for (int i = 0; i < r; ++i) x -= sm.M[r][i] * ucol[i];
        ucol[r] = x;
      }
#pragma unroll
      for (int r = 0; r < T; ++r) sm.u[r][j] = ucol[r];
    }
    __syncthreads();

    // Outputs O = Qt S0 + P U.
    for (int e = tid; e < T * W; e += NT) {
      const int r = e / W, j = e % W;
      if (r >= L) continue;
      float o = 0.f;
#pragma unroll 8
      for (int c = 0; c < DK; ++c) o += sm.q[r][c] * sm.eg[r][c] * sm.S[c][j];
      for (int i = 0; i <= r; ++i) o += sm.P[r][i] * sm.u[i][j];
      out[((size_t)(c0 + r) * H + h) * DV + col0 + j] = from_f32<TIn>(o);
    }
    __syncthreads();

    // State carry S = Diag(exp(Gam_L)) S0 + Kh^T U (each thread owns its entries).
    for (int e = tid; e < DK * W; e += NT) {
      const int c = e / W, j = e % W;
      float s = sm.eg[T - 1][c] * sm.S[c][j];
#pragma unroll
      for (int r = 0; r < T; ++r) s += sm.k[r][c] * sm.eh[r][c] * sm.u[r][j];
      sm.S[c][j] = s;
    }

    done += L;
    if (ckpt_interval > 0 && done % ckpt_interval == 0) store_state(ckpt_states, ck_slot++);
    while (pi < pe && positions[pi] <= done) store_state(pos_states, pi++);
  }
  while (pi < pe) store_state(pos_states, pi++);   // positions past the end: final state
  __syncthreads();
  if (final_state)
    for (int e = tid; e < DK * W; e += NT) {
      const int c = e / W, j = e % W;
      final_state[state_off + (size_t)c * DV + col0 + j] = sm.S[c][j];
    }
}

template <int DK, typename TIn>
static cudaError_t launch_simt_t(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *init, const int32_t *cu,
                                 void *out, float *fin, int64_t interval, float *ck,
                                 const int32_t *pos_cu, const int32_t *positions,
                                 float *pos_states, int N, int H, int DV, cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem<DK>);
  auto kern = prefill_simt_kernel<DK, TIn>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)((int64_t)N * H), (unsigned)(DV / kSimtSlice));
  kern<<<grid, kSimtThreads, smem, stream>>>((const TIn *)q, (const TIn *)k, (const TIn *)v, g,
                                             beta, init, cu, (TIn *)out, fin, interval, ck,
                                             pos_cu, positions, pos_states, H, DV);
  return cudaGetLastError();
}

cudaError_t launch_prefill_simt(int dtype, int dk, int dv, const void *q, const void *k,
                                const void *v, const float *g, const float *beta,
                                const float *init, const int32_t *cu, void *out, float *fin,
                                int64_t interval, float *ck, const int32_t *pos_cu,
                                const int32_t *positions, float *pos_states, int N, int H,
                                cudaStream_t stream) {
  if (dv % kSimtSlice != 0) return cudaErrorInvalidValue;
#define KDA_SIMT(DK_)                                                                        \
  if (dk == DK_) {                                                                           \
    if (dtype == KDA_DTYPE_BF16)                                                             \
      return launch_simt_t<DK_, __nv_bfloat16>(q, k, v, g, beta, init, cu, out, fin,         \
                                               interval, ck, pos_cu, positions, pos_states,  \
                                               N, H, dv, stream);                            \
    return launch_simt_t<DK_, float>(q, k, v, g, beta, init, cu, out, fin, interval, ck,     \
                                     pos_cu, positions, pos_states, N, H, dv, stream);       \
  }
  KDA_SIMT(32) KDA_SIMT(64) KDA_SIMT(128)
#undef KDA_SIMT
  return cudaErrorInvalidValue;
}

}  // namespace kda
