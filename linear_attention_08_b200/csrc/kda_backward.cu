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
// Column j of S only ever meets column j of dS, v, do, u and du: the
// recurrence and its reverse split by value columns.  Only dq, dk, dg and
// dbeta sum over columns, and those sums are linear.  So one CTA of 128
// threads takes one (sequence, head, slice of 32 value columns): lane j owns
// column j of the slice, warp w the rows [w D_k/4, (w+1) D_k/4), and the
// thread keeps its D_k/4 entries of S and of dS in registers.  Column sums
// (y, du) cross the four warps through a small shared array; row sums (the
// parts of dq, dk, dg) are reduce-scattered across the warp's lanes by
// shuffles, so each lane ends with one row's sum.  Slice 0 writes dq, dk, dg,
// dbeta; slices 1.. write their parts to the workspace, and a second kernel
// adds them in slice order.
//
// A forward sweep stores the state at the start of every block of kBlk
// tokens in the workspace.  The reverse sweep walks the blocks backwards:
// it reloads the block's state, replays the block once (keeping the states
// before its middle tokens in shared memory, the last one in registers), and
// then takes the backward steps from the last token down.
#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kBThreads = 128;
constexpr int kBlk = 4;       // tokens between stored states
constexpr int kCols = 32;     // value columns per CTA
constexpr unsigned kFull = 0xffffffffu;

struct BwdArgs {
  const void *q, *k, *v;
  const float *g, *beta, *init;
  const int32_t *cu;
  const float *dout, *dfin;
  float *dq, *dk, *dv, *dg, *dbeta, *dinit;
  float *ckpt;        // stored states
  float *part;        // row-sum parts of slices 1..NS-1 (NS > 1 only)
  int64_t T;          // total tokens
  int H;
};

template <typename TIn>
__device__ __forceinline__ float ld_in(const void *p, size_t i) {
  return to_f32(reinterpret_cast<const TIn *>(p)[i]);
}

// Sum of v[i] over the 32 lanes for every i < M, scattered: on return, lane L
// holds the sum for row i = L >> (5 - log2 M).  Recursive halving: at each
// level a lane keeps one half of its values and adds its partner's copy of
// that half, so a level of m values costs m/2 shuffles.
template <int M>
__device__ __forceinline__ float reduce_scatter(float (&v)[M], int lane) {
#pragma unroll
  for (int lvl = 0; (M >> lvl) > 1; ++lvl) {
    const int half = M >> (lvl + 1), o = 16 >> lvl;
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, o);
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = 16 / M; o >= 1; o >>= 1) r += __shfl_xor_sync(kFull, r, o);
  return r;
}

template <int M> struct Log2 { static constexpr int value = 1 + Log2<M / 2>::value; };
template <> struct Log2<1> { static constexpr int value = 0; };

// Shared memory, in floats.
template <int Dk>
struct BwdSmem {
  static constexpr int RPW = Dk / 4;
  static constexpr int TK = 0;                        // k        [kBlk][Dk]
  static constexpr int TA = TK + kBlk * Dk;           // alpha    [kBlk][Dk]
  static constexpr int TQ = TA + kBlk * Dk;           // q        [kBlk][Dk]
  static constexpr int TV = TQ + kBlk * Dk;           // v slice  [kBlk][32]
  static constexpr int TD = TV + kBlk * kCols;        // do slice [kBlk][32]
  static constexpr int TB = TD + kBlk * kCols;        // beta     [kBlk] (padded to 4)
  static constexpr int PY = TB + 4;                   // y parts  [2][4][32]
  static constexpr int PD = PY + 2 * 4 * kCols;       // du parts [2][4][32]
  static constexpr int ST = PD + 2 * 4 * kCols;       // states   [kBlk-2][RPW][128]
  static constexpr int TOTAL = ST + (kBlk - 2) * RPW * kBThreads;
};

template <typename TIn, int Dk, int Dv>
__global__ void __launch_bounds__(kBThreads, 4) backward_kernel(const BwdArgs a) {
  using L = BwdSmem<Dk>;
  constexpr int RPW = L::RPW, NS = Dv / kCols, DD = Dk * Dv;
  constexpr int SHIFT = 5 - Log2<RPW>::value;
  extern __shared__ __align__(16) float smem[];
  const int tid = threadIdx.x, w = tid >> 5, j = tid & 31;
  const int H = a.H;
  const int slice = blockIdx.x % NS, unit = blockIdx.x / NS, n = unit / H, h = unit % H;
  const int col = slice * kCols + j;
  const int row0 = w * RPW;
  const int64_t t_begin = a.cu[n], T = (int64_t)a.cu[n + 1] - t_begin;
  const int64_t nb = (T + kBlk - 1) / kBlk;
  int64_t before = 0;   // stored states of all earlier sequences, per head
  for (int m = 0; m < n; ++m) before += ((int64_t)a.cu[m + 1] - a.cu[m] + kBlk - 1) / kBlk;
  float *ck = a.ckpt + ((size_t)before * H + (size_t)h * nb) * DD;

  float *tk = smem + L::TK, *ta = smem + L::TA, *tq = smem + L::TQ;
  float *tv = smem + L::TV, *tdo = smem + L::TD, *tb = smem + L::TB;
  float *py = smem + L::PY, *pdu = smem + L::PD, *st = smem + L::ST;

  // Where this slice's row-sum parts go: the outputs for slice 0, else the workspace.
  const size_t n_k = (size_t)a.T * H * Dk;
  float *oq = a.dq, *okk = a.dk, *og = a.dg, *ob = a.dbeta;
  if (slice > 0) {
    const size_t s1 = slice - 1;
    oq = a.part + s1 * n_k;
    okk = a.part + (NS - 1) * n_k + s1 * n_k;
    og = a.part + 2 * (NS - 1) * n_k + s1 * n_k;
    ob = a.part + 3 * (NS - 1) * n_k + s1 * (size_t)a.T * H;
  }

  float S[RPW], dS[RPW];
  int par = 0;

  auto load_tokens = [&](int64_t t_lo, int cnt, bool full) {
    for (int e = tid; e < cnt * Dk; e += kBThreads) {
      const int s = e / Dk, c = e - s * Dk;
      const size_t ix = ((size_t)(t_begin + t_lo + s) * H + h) * Dk + c;
      tk[s * Dk + c] = ld_in<TIn>(a.k, ix);
      ta[s * Dk + c] = __expf(a.g[ix]);
      if (full) tq[s * Dk + c] = ld_in<TIn>(a.q, ix);
    }
    for (int e = tid; e < cnt * kCols; e += kBThreads) {
      const int s = e >> 5, jj = e & 31;
      const size_t ix = ((size_t)(t_begin + t_lo + s) * H + h) * Dv + slice * kCols + jj;
      tv[s * kCols + jj] = ld_in<TIn>(a.v, ix);
      if (full) tdo[s * kCols + jj] = a.dout[ix];
    }
    if (tid < cnt) tb[tid] = a.beta[(size_t)(t_begin + t_lo + tid) * H + h];
  };
  auto load_state = [&](int64_t b) {
    const float *src = ck + (size_t)b * DD;
#pragma unroll
    for (int i = 0; i < RPW; ++i) S[i] = src[(row0 + i) * Dv + col];
  };
  // One forward step of token slot s: S <- Diag(alpha) S + k u^T.  The warps'
  // parts of y_j = sum_c alpha_c k_c S_cj meet in py.
  auto fwd_step = [&](int s) {
    const float *k_s = tk + s * Dk + row0, *a_s = ta + s * Dk + row0;
    float pa = 0.f;
#pragma unroll
    for (int i = 0; i < RPW; i += 4) {
      const float4 k4 = *reinterpret_cast<const float4 *>(k_s + i);
      const float4 a4 = *reinterpret_cast<const float4 *>(a_s + i);
      pa = fmaf(a4.x * k4.x, S[i], pa);
      pa = fmaf(a4.y * k4.y, S[i + 1], pa);
      pa = fmaf(a4.z * k4.z, S[i + 2], pa);
      pa = fmaf(a4.w * k4.w, S[i + 3], pa);
    }
    float *pp = py + par * 4 * kCols;
    pp[w * kCols + j] = pa;
    __syncthreads();
    const float y = (pp[j] + pp[kCols + j]) + (pp[2 * kCols + j] + pp[3 * kCols + j]);
    par ^= 1;
    const float u = tb[s] * (tv[s * kCols + j] - y);
#pragma unroll
    for (int i = 0; i < RPW; i += 4) {
      const float4 k4 = *reinterpret_cast<const float4 *>(k_s + i);
      const float4 a4 = *reinterpret_cast<const float4 *>(a_s + i);
      S[i] = fmaf(a4.x, S[i], k4.x * u);
      S[i + 1] = fmaf(a4.y, S[i + 1], k4.y * u);
      S[i + 2] = fmaf(a4.z, S[i + 2], k4.z * u);
      S[i + 3] = fmaf(a4.w, S[i + 3], k4.w * u);
    }
  };
  // Backward step of token slot s (token t): S holds S_{t-1}, dS the gradient
  // w.r.t. S_t from later tokens.
  auto bwd_step = [&](int s, int64_t t) {
    const float *k_s = tk + s * Dk + row0, *a_s = ta + s * Dk + row0, *q_s = tq + s * Dk + row0;
    const float doj = tdo[s * kCols + j];
    float pa = 0.f, pd = 0.f;
#pragma unroll
    for (int i = 0; i < RPW; i += 4) {
      const float4 k4 = *reinterpret_cast<const float4 *>(k_s + i);
      const float4 a4 = *reinterpret_cast<const float4 *>(a_s + i);
      const float4 q4 = *reinterpret_cast<const float4 *>(q_s + i);
      pa = fmaf(a4.x * k4.x, S[i], pa);
      pa = fmaf(a4.y * k4.y, S[i + 1], pa);
      pa = fmaf(a4.z * k4.z, S[i + 2], pa);
      pa = fmaf(a4.w * k4.w, S[i + 3], pa);
      dS[i] = fmaf(q4.x, doj, dS[i]);
      dS[i + 1] = fmaf(q4.y, doj, dS[i + 1]);
      dS[i + 2] = fmaf(q4.z, doj, dS[i + 2]);
      dS[i + 3] = fmaf(q4.w, doj, dS[i + 3]);
      pd = fmaf(k4.x, dS[i], pd);
      pd = fmaf(k4.y, dS[i + 1], pd);
      pd = fmaf(k4.z, dS[i + 2], pd);
      pd = fmaf(k4.w, dS[i + 3], pd);
    }
    float *pp = py + par * 4 * kCols, *pq = pdu + par * 4 * kCols;
    pp[w * kCols + j] = pa;
    pq[w * kCols + j] = pd;
    __syncthreads();
    const float y = (pp[j] + pp[kCols + j]) + (pp[2 * kCols + j] + pp[3 * kCols + j]);
    const float du = (pq[j] + pq[kCols + j]) + (pq[2 * kCols + j] + pq[3 * kCols + j]);
    par ^= 1;
    const float bt = tb[s], vj = tv[s * kCols + j];
    const float u = bt * (vj - y);
    const size_t th = (size_t)(t_begin + t) * H + h;
    if (w == 0) a.dv[th * Dv + col] = bt * du;
    // this slice's parts of du.(v - y) and u.do
    float db = du * (vj - y), ud = u * doj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      db += __shfl_xor_sync(kFull, db, o);
      ud += __shfl_xor_sync(kFull, ud, o);
    }
    if (tid == 0) ob[th] = db;
    // row sums over the slice: r1 = S do, r3 = S du, r2 = dS u, r4 = sum_j dS_cj S_cj
    float tmp[RPW];
#pragma unroll
    for (int i = 0; i < RPW; ++i) tmp[i] = S[i] * doj;
    const float r1 = reduce_scatter<RPW>(tmp, j);
#pragma unroll
    for (int i = 0; i < RPW; ++i) tmp[i] = S[i] * du;
    const float r3 = reduce_scatter<RPW>(tmp, j);
#pragma unroll
    for (int i = 0; i < RPW; ++i) tmp[i] = dS[i] * u;
    const float r2 = reduce_scatter<RPW>(tmp, j);
#pragma unroll
    for (int i = 0; i < RPW; ++i) tmp[i] = dS[i] * S[i];
    const float r4 = reduce_scatter<RPW>(tmp, j);
    if ((j & ((1 << SHIFT) - 1)) == 0) {
      const int c = row0 + (j >> SHIFT);
      const float al = ta[s * Dk + c], kc = tk[s * Dk + c];
      const size_t o = th * Dk + c;
      // S_t = Diag(alpha) S_{t-1} + k u^T, so S_t do = alpha (S_{t-1} do) + k (u . do)
      oq[o] = fmaf(al, r1, kc * ud);
      okk[o] = r2 - bt * al * r3;
      og[o] = al * (r4 - bt * kc * r3);
    }
    // dS <- Diag(alpha) (dS - beta k du^T)
    const float nbd = -bt * du;
#pragma unroll
    for (int i = 0; i < RPW; i += 4) {
      const float4 k4 = *reinterpret_cast<const float4 *>(k_s + i);
      const float4 a4 = *reinterpret_cast<const float4 *>(a_s + i);
      dS[i] = a4.x * fmaf(k4.x, nbd, dS[i]);
      dS[i + 1] = a4.y * fmaf(k4.y, nbd, dS[i + 1]);
      dS[i + 2] = a4.z * fmaf(k4.z, nbd, dS[i + 2]);
      dS[i + 3] = a4.w * fmaf(k4.w, nbd, dS[i + 3]);
    }
  };

  // ---------------- forward sweep: the state at the start of every block ----------------
#pragma unroll
  for (int i = 0; i < RPW; ++i)
    S[i] = a.init ? a.init[(size_t)unit * DD + (row0 + i) * Dv + col] : 0.f;
  for (int64_t b = 0; b < nb; ++b) {
    const int64_t t_lo = b * kBlk;
    const int cnt = (int)((T - t_lo) < kBlk ? (T - t_lo) : kBlk);
    float *dst = ck + (size_t)b * DD;
#pragma unroll
    for (int i = 0; i < RPW; ++i) dst[(row0 + i) * Dv + col] = S[i];
    __syncthreads();   // the previous block's tokens are no longer read
    load_tokens(t_lo, cnt, false);
    __syncthreads();
    for (int s = 0; s < cnt; ++s) fwd_step(s);
  }

  // ---------------- reverse sweep ----------------
#pragma unroll
  for (int i = 0; i < RPW; ++i)
    dS[i] = a.dfin ? a.dfin[(size_t)unit * DD + (row0 + i) * Dv + col] : 0.f;
  for (int64_t b = nb - 1; b >= 0; --b) {
    const int64_t t_lo = b * kBlk;
    const int cnt = (int)((T - t_lo) < kBlk ? (T - t_lo) : kBlk);
    __syncthreads();
    load_tokens(t_lo, cnt, true);
    load_state(b);
    __syncthreads();
    // replay: S becomes the state before token slot cnt-1; the states before
    // slots 1 .. cnt-2 are kept, each thread its own entries
    for (int s = 0; s + 1 < cnt; ++s) {
      fwd_step(s);
      if (s + 1 < cnt - 1) {
        float *slot = st + (size_t)s * RPW * kBThreads;
#pragma unroll
        for (int i = 0; i < RPW; ++i) slot[i * kBThreads + tid] = S[i];
      }
    }
    for (int s = cnt - 1; s >= 0; --s) {
      if (s < cnt - 1) {
        if (s >= 1) {
          const float *slot = st + (size_t)(s - 1) * RPW * kBThreads;
#pragma unroll
          for (int i = 0; i < RPW; ++i) S[i] = slot[i * kBThreads + tid];
        } else {
          load_state(b);
        }
      }
      bwd_step(s, t_lo + s);
    }
  }
  if (a.dinit)
#pragma unroll
    for (int i = 0; i < RPW; ++i) a.dinit[(size_t)unit * DD + (row0 + i) * Dv + col] = dS[i];
}

// dq, dk, dg, dbeta += the parts of slices 1..ns-1, in slice order.
__global__ void __launch_bounds__(256) backward_sum_kernel(float *__restrict__ dq, float *__restrict__ dk,
                                                           float *__restrict__ dg, float *__restrict__ dbeta,
                                                           const float *__restrict__ part, int64_t n_k,
                                                           int64_t n_b, int extra) {
  const int64_t n4 = n_k / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  float4 *outs[3] = {reinterpret_cast<float4 *>(dq), reinterpret_cast<float4 *>(dk),
                     reinterpret_cast<float4 *>(dg)};
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += stride) {
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      float4 acc = outs[m][e];
      for (int s = 0; s < extra; ++s) {
        const float4 p = reinterpret_cast<const float4 *>(part + ((size_t)m * extra + s) * n_k)[e];
        acc.x += p.x;
        acc.y += p.y;
        acc.z += p.z;
        acc.w += p.w;
      }
      outs[m][e] = acc;
    }
  }
  const float *pb = part + (size_t)3 * extra * n_k;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n_b; e += stride) {
    float acc = dbeta[e];
    for (int s = 0; s < extra; ++s) acc += pb[(size_t)s * n_b + e];
    dbeta[e] = acc;
  }
}

}  // namespace

size_t backward_smem_bytes(int Dk) {
  switch (Dk) {
    case 32: return sizeof(float) * BwdSmem<32>::TOTAL;
    case 64: return sizeof(float) * BwdSmem<64>::TOTAL;
    default: return sizeof(float) * BwdSmem<128>::TOTAL;
  }
}

static size_t ckpt_floats(int N, int H, int64_t T, int Dk, int Dv) {
  // sum over sequences of ceil(T_n / kBlk) <= (T + (kBlk - 1) N) / kBlk
  return (size_t)((T + (int64_t)(kBlk - 1) * N) / kBlk) * H * Dk * Dv;
}

size_t backward_workspace_bytes(int N, int H, int64_t T, int Dk, int Dv) {
  const size_t extra = (size_t)(Dv / kCols - 1);
  return sizeof(float) * (ckpt_floats(N, H, T, Dk, Dv) + extra * (size_t)T * H * (3 * (size_t)Dk + 1));
}

template <typename TIn, int DK, int DV>
static cudaError_t launch_backward_t(const BwdArgs &args, int N, cudaStream_t stream) {
  const size_t smem = backward_smem_bytes(DK);
  cudaError_t e = cudaFuncSetAttribute(backward_kernel<TIn, DK, DV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  constexpr int NS = DV / kCols;
  const unsigned grid = (unsigned)((int64_t)N * args.H * NS);
  backward_kernel<TIn, DK, DV><<<grid, kBThreads, smem, stream>>>(args);
  e = cudaGetLastError();
  if (e != cudaSuccess || NS == 1 || args.T == 0) return e;
  const int64_t n_k = args.T * args.H * DK;
  const int64_t n4 = n_k / 4;
  const unsigned sum_grid = (unsigned)((n4 + 255) / 256 < 148 * 8 ? (n4 + 255) / 256 : 148 * 8);
  backward_sum_kernel<<<sum_grid, 256, 0, stream>>>(args.dq, args.dk, args.dg, args.dbeta, args.part,
                                                    n_k, args.T * args.H, NS - 1);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_backward_d(const BwdArgs &args, int Dk, int Dv, int N, cudaStream_t stream) {
#define KDA_BWD(DK_, DV_) \
  if (Dk == DK_ && Dv == DV_) return launch_backward_t<TIn, DK_, DV_>(args, N, stream);
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
                            int Dv, int64_t T, cudaStream_t stream) {
  float *part = ws + ckpt_floats(N, H, T, Dk, Dv);
  const BwdArgs args{q, k, v, g, beta, init, cu, dout, dfin, dq, dk, dv, dg, dbeta, dinit, ws, part,
                     T, H};
  if (dtype == KDA_DTYPE_BF16) return launch_backward_d<__nv_bfloat16>(args, Dk, Dv, N, stream);
  return launch_backward_d<float>(args, Dk, Dv, N, stream);
}

}  // namespace kda
