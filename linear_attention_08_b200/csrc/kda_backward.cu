// Backward pass of the KDA recurrence (training direction), FP32 SIMT.
//
// The pages give no detail of the backward pass; it is the reverse of the
// forward recurrence ("LLM - Semianalysis, Kimi K3 아키텍처", Background: the
// gated delta rule S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T,
// o_t = S_t^T q_t).  Per token, with P = Diag(alpha_t) S_{t-1},
// y = P^T k_t, u = beta_t (v_t - y), S_t = P + k_t u^T, and dS the gradient
// with respect to S_t from later tokens:
//
//   dS   += q_t do_t^T                 dq_t   = S_t do_t
//   du    = dS^T k_t                   dk_t   = dS u - beta_t P du
//   dbeta = du . (v_t - y)             dv_t   = beta_t du
//   dg_c  = alpha_c sum_j (dS - beta k du^T)_cj S_{t-1,cj}
//   dS   <- Diag(alpha_t) (dS - beta_t k_t du^T)       (gradient w.r.t. S_{t-1})
//
// One CTA (256 threads) per (sequence, head).  A forward sweep stores the
// state at every 8th token in the workspace; the reverse sweep rebuilds
// S_{t-1} for each token from the nearest stored state (at most 7 forward
// steps) and applies the step above.  The state, its copy at the block start
// and dS live in shared memory with a padded row stride (D_v + 1 floats), so
// that both row-wise and column-wise passes are free of bank conflicts.
#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kBThreads = 256;
constexpr int kBlk = 8;       // tokens between stored states
constexpr int kMaxD = 128;

struct BwdArgs {
  const void *q, *k, *v;
  const float *g, *beta, *init;
  const int32_t *cu;
  const float *dout, *dfin;
  float *dq, *dk, *dv, *dg, *dbeta, *dinit;
  float *ws;
  int H;
};

template <typename TIn>
__device__ __forceinline__ float ld_in(const void *p, size_t i) {
  return to_f32(reinterpret_cast<const TIn *>(p)[i]);
}

template <typename TIn, int Dk, int Dv>
__global__ void __launch_bounds__(kBThreads, 1) backward_kernel(const BwdArgs a) {
  extern __shared__ float smem[];
  const int H = a.H;
  constexpr int ld = Dv + 1;
  float *S = smem;                        // [Dk][Dv+1] working state (S_{t-1} after the replay)
  float *dS = S + Dk * ld;                // [Dk][Dv+1]
  float *S0 = dS + Dk * ld;               // [Dk][Dv]  stored state of the current block
  float *vk = S0 + Dk * Dv;               // k_t
  float *vq = vk + kMaxD;                 // q_t
  float *va = vq + kMaxD;                 // alpha_t
  float *vv = va + kMaxD;                 // v_t
  float *vdo = vv + kMaxD;                // do_t
  float *vy = vdo + kMaxD;                // y
  float *vu = vy + kMaxD;                 // u
  float *vdu = vu + kMaxD;                // du
  float *part = vdu + kMaxD;              // [4][kBThreads] partial sums
  float *scal = part + 4 * kBThreads;     // [4]: beta, u.do, dbeta partials

  const int tid = threadIdx.x;
  const int unit = blockIdx.x, n = unit / H, h = unit % H;
  const int64_t t_begin = a.cu[n], T = (int64_t)a.cu[n + 1] - t_begin;
  const int64_t nb = (T + kBlk - 1) / kBlk;
  // this unit's stored states: blocks of all earlier sequences, then h * nb
  int64_t before = 0;
  for (int m = 0; m < n; ++m) before += ((int64_t)a.cu[m + 1] - a.cu[m] + kBlk - 1) / kBlk;
  float *wsu = a.ws + ((size_t)before * H + (size_t)h * nb) * Dk * Dv;
  constexpr int DD = Dk * Dv;

  // Column passes and elementwise passes: thread (j, part) takes column j of
  // rows c = part, part + cp, ...; row passes: thread (c, part) takes row c
  // at columns j = part, part + rp, ...
  constexpr int cp = kBThreads / Dv;      // 2, 4 or 8
  const int cj = tid % Dv, cpart = tid / Dv;
  constexpr int rp = kBThreads / Dk;
  const int rc = tid % Dk, rpart = tid / Dk;

  auto load_token = [&](int64_t t, bool full) {
    const size_t tk = ((size_t)(t_begin + t) * H + h);
    if (tid < Dk) {
      vk[tid] = ld_in<TIn>(a.k, tk * Dk + tid);
      va[tid] = __expf(a.g[tk * Dk + tid]);
      if (full) vq[tid] = ld_in<TIn>(a.q, tk * Dk + tid);
    }
    if (tid < Dv) {
      vv[tid] = ld_in<TIn>(a.v, tk * Dv + tid);
      if (full) vdo[tid] = a.dout[tk * Dv + tid];
    }
    if (tid == 0) scal[0] = a.beta[tk];
  };
  // y_j = sum_c alpha_c k_c S_cj  (S = S_{t-1}), into vy; u into vu.
  auto form_y_u = [&]() {
    float s = 0.f;
    for (int c = cpart; c < Dk; c += cp) s = fmaf(va[c] * vk[c], S[c * ld + cj], s);
    part[tid] = s;
    __syncthreads();
    if (tid < Dv) {
      float y = 0.f;
      for (int p = 0; p < cp; ++p) y += part[p * Dv + tid];
      vy[tid] = y;
      vu[tid] = scal[0] * (vv[tid] - y);
    }
    __syncthreads();
  };
  // One forward step on S: S <- Diag(alpha) S + k u^T.
  auto forward_step = [&](int64_t t) {
    load_token(t, false);
    __syncthreads();
    form_y_u();
    const float uj = vu[cj];
#pragma unroll
    for (int c = cpart; c < Dk; c += cp) S[c * ld + cj] = fmaf(va[c], S[c * ld + cj], vk[c] * uj);
    __syncthreads();
  };

  // ---------------- forward sweep: states at every 8th token ----------------
#pragma unroll
  for (int c = cpart; c < Dk; c += cp)
    S[c * ld + cj] = a.init ? a.init[(size_t)unit * DD + c * Dv + cj] : 0.f;
  __syncthreads();
  for (int64_t t = 0; t < T; ++t) {
    if (t % kBlk == 0) {
      float *dst = wsu + (size_t)(t / kBlk) * DD;
#pragma unroll
      for (int c = cpart; c < Dk; c += cp) dst[c * Dv + cj] = S[c * ld + cj];
    }
    forward_step(t);
  }

  // ---------------- reverse sweep ----------------
#pragma unroll
  for (int c = cpart; c < Dk; c += cp)
    dS[c * ld + cj] = a.dfin ? a.dfin[(size_t)unit * DD + c * Dv + cj] : 0.f;
  __syncthreads();
  for (int64_t b = nb - 1; b >= 0; --b) {
    const int64_t t_lo = b * kBlk, t_hi = (t_lo + kBlk < T) ? t_lo + kBlk : T;
    const float *src = wsu + (size_t)b * DD;
#pragma unroll
    for (int c = cpart; c < Dk; c += cp) S0[c * Dv + cj] = src[c * Dv + cj];
    __syncthreads();
    for (int64_t t = t_hi - 1; t >= t_lo; --t) {
      // rebuild S_{t-1} from the block's stored state
#pragma unroll
      for (int c = cpart; c < Dk; c += cp) S[c * ld + cj] = S0[c * Dv + cj];
      __syncthreads();
      for (int64_t r = t_lo; r < t; ++r) forward_step(r);
      // ---- backward step of token t ----
      load_token(t, true);
      __syncthreads();
      form_y_u();
      // dS += q do^T
      {
        const float doj = vdo[cj];
#pragma unroll
        for (int c = cpart; c < Dk; c += cp) dS[c * ld + cj] = fmaf(vq[c], doj, dS[c * ld + cj]);
      }
      __syncthreads();
      // du_j = sum_c k_c dS_cj
      {
        float s = 0.f;
        for (int c = cpart; c < Dk; c += cp) s = fmaf(vk[c], dS[c * ld + cj], s);
        part[tid] = s;
      }
      __syncthreads();
      const float bt = scal[0];
      if (tid < Dv) {
        float du = 0.f;
        for (int p = 0; p < cp; ++p) du += part[p * Dv + tid];
        vdu[tid] = du;
        a.dv[((size_t)(t_begin + t) * H + h) * Dv + tid] = bt * du;
      }
      __syncthreads();
      // dbeta = du . (v - y) and u . do (warp 0)
      if (tid < 32) {
        float db = 0.f, ud = 0.f;
        for (int j = tid; j < Dv; j += 32) {
          db = fmaf(vdu[j], vv[j] - vy[j], db);
          ud = fmaf(vu[j], vdo[j], ud);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          db += __shfl_xor_sync(0xffffffffu, db, o);
          ud += __shfl_xor_sync(0xffffffffu, ud, o);
        }
        if (tid == 0) {
          a.dbeta[(size_t)(t_begin + t) * H + h] = db;
          scal[1] = ud;
        }
      }
      // row sums: r1 = S do, r2 = dS u, r3 = S du, r4 = sum_j dS_cj S_cj
      {
        float r1 = 0.f, r2 = 0.f, r3 = 0.f, r4 = 0.f;
        for (int j = rpart; j < Dv; j += rp) {
          const float s = S[rc * ld + j], d = dS[rc * ld + j];
          r1 = fmaf(s, vdo[j], r1);
          r2 = fmaf(d, vu[j], r2);
          r3 = fmaf(s, vdu[j], r3);
          r4 = fmaf(d, s, r4);
        }
        part[tid] = r1;
        part[kBThreads + tid] = r2;
        part[2 * kBThreads + tid] = r3;
        part[3 * kBThreads + tid] = r4;
      }
      __syncthreads();
      if (tid < Dk) {
        float r1 = 0.f, r2 = 0.f, r3 = 0.f, r4 = 0.f;
        for (int p = 0; p < rp; ++p) {
          r1 += part[p * Dk + tid];
          r2 += part[kBThreads + p * Dk + tid];
          r3 += part[2 * kBThreads + p * Dk + tid];
          r4 += part[3 * kBThreads + p * Dk + tid];
        }
        const float al = va[tid], kc = vk[tid];
        const size_t o = ((size_t)(t_begin + t) * H + h) * Dk + tid;
        // S_t = Diag(alpha) S_{t-1} + k u^T, so S_t do = alpha (S do) + k (u . do)
        a.dq[o] = fmaf(al, r1, kc * scal[1]);
        a.dk[o] = r2 - bt * al * r3;
        a.dg[o] = al * (r4 - bt * kc * r3);
      }
      // dS <- Diag(alpha) (dS - beta k du^T)
      {
        const float duj = vdu[cj];
#pragma unroll
        for (int c = cpart; c < Dk; c += cp)
          dS[c * ld + cj] = va[c] * fmaf(-bt * vk[c], duj, dS[c * ld + cj]);
      }
      __syncthreads();
    }
  }
  if (a.dinit)
#pragma unroll
    for (int c = cpart; c < Dk; c += cp) a.dinit[(size_t)unit * DD + c * Dv + cj] = dS[c * ld + cj];
}

}  // namespace

size_t backward_smem_bytes(int Dk, int Dv) {
  return sizeof(float) * ((size_t)2 * Dk * (Dv + 1) + (size_t)Dk * Dv + 8 * kMaxD + 4 * kBThreads + 4);
}

size_t backward_workspace_bytes(int N, int H, int64_t T, int Dk, int Dv) {
  return sizeof(float) * (size_t)((T + (int64_t)(kBlk - 1) * N) / kBlk) * H * Dk * Dv;
}

template <typename TIn, int DK, int DV>
static cudaError_t launch_backward_t(const BwdArgs &args, unsigned grid, cudaStream_t stream) {
  const size_t smem = backward_smem_bytes(DK, DV);
  cudaError_t e = cudaFuncSetAttribute(backward_kernel<TIn, DK, DV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  backward_kernel<TIn, DK, DV><<<grid, kBThreads, smem, stream>>>(args);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_backward_d(const BwdArgs &args, int Dk, int Dv, unsigned grid,
                                     cudaStream_t stream) {
#define KDA_BWD(DK_, DV_) \
  if (Dk == DK_ && Dv == DV_) return launch_backward_t<TIn, DK_, DV_>(args, grid, stream);
  KDA_BWD(32, 32) KDA_BWD(32, 64) KDA_BWD(32, 128)
  KDA_BWD(64, 32) KDA_BWD(64, 64) KDA_BWD(64, 128)
  KDA_BWD(128, 32) KDA_BWD(128, 64) KDA_BWD(128, 128)
#undef KDA_BWD
  return cudaErrorInvalidValue;
}

cudaError_t launch_backward(int dtype, const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *init, const int32_t *cu,
                            const float *dout, const float *dfin, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *dinit, float *ws, int N, int H, int Dk,
                            int Dv, cudaStream_t stream) {
  const BwdArgs args{q, k, v, g, beta, init, cu, dout, dfin, dq, dk, dv, dg, dbeta, dinit, ws, H};
  const unsigned grid = (unsigned)((int64_t)N * H);
  if (dtype == KDA_DTYPE_BF16) return launch_backward_d<__nv_bfloat16>(args, Dk, Dv, grid, stream);
  return launch_backward_d<float>(args, Dk, Dv, grid, stream);
}

}  // namespace kda
