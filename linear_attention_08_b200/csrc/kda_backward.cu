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
// threads takes one (sequence, head, slice of 32 value columns).  Warp w owns
// the rows [w D_k/4, (w+1) D_k/4); each thread keeps a tile of D_k/16 rows x
// 4 columns of S and of dS in registers.  Column sums (y, du) are summed over
// the tile's rows, reduce-scattered over the warp's row groups, and the four
// warps' parts meet in a small shared array (one barrier per step).  Row sums
// (the parts of dq, dk, dg) are summed over the tile's 4 columns and
// reduce-scattered over the warp's 8 column groups, so each lane ends with one
// row's sum.  Slice 0 writes dq, dk, dg, dbeta; slices 1.. write their parts
// to the workspace, and a second kernel adds them in slice order.
//
// A forward sweep stores the state at the start of every block of kBlk
// tokens in the workspace.  The reverse sweep walks the blocks backwards:
// it reloads the block's state, replays the block once (keeping the states
// before its middle tokens in shared memory, the last one in registers), and
// then takes the backward steps from the last token down.  The next block's
// tokens are staged by cp.async while the current block computes.
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

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Reduce-scatter across lanes: v[i] (i < M) is summed over the lanes that
// differ in the lane bits OHI, OHI/2, ..., OLO; on return the lane holds the
// sum for one i, i = the lane's bits OHI .. (OHI >> (log2 M - 1)) read as a
// binary number (highest first).  Recursive halving: at each level a lane
// keeps one half of its values and adds its partner's copy of that half, so
// a level of m values costs m/2 shuffles; bits below the halving levels are
// summed by plain butterflies.
template <int M, int OHI, int OLO>
__device__ __forceinline__ float reduce_scatter(float (&v)[M], int lane) {
#pragma unroll
  for (int lvl = 0; (M >> lvl) > 1; ++lvl) {
    const int half = M >> (lvl + 1), o = OHI >> lvl;
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
  for (int o = OHI / M; o >= OLO; o >>= 1) r += __shfl_xor_sync(kFull, r, o);
  return r;
}

template <int M> struct Log2 { static constexpr int value = 1 + Log2<M / 2>::value; };
template <> struct Log2<1> { static constexpr int value = 0; };

// RT consecutive floats from shared memory (RT in {2, 4, 8}, aligned to RT floats).
template <int RT>
__device__ __forceinline__ void lds_rows(const float *p, float (&o)[RT]) {
  if constexpr (RT % 4 == 0) {
#pragma unroll
    for (int i = 0; i < RT; i += 4) {
      const float4 x = *reinterpret_cast<const float4 *>(p + i);
      o[i] = x.x;
      o[i + 1] = x.y;
      o[i + 2] = x.z;
      o[i + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < RT; i += 2) {
      const float2 x = *reinterpret_cast<const float2 *>(p + i);
      o[i] = x.x;
      o[i + 1] = x.y;
    }
  }
}

__device__ __forceinline__ void lds4(const float *p, float (&o)[4]) {
  const float4 x = *reinterpret_cast<const float4 *>(p);
  o[0] = x.x;
  o[1] = x.y;
  o[2] = x.z;
  o[3] = x.w;
}

// Shared memory, in floats.  ES is the byte size of a q, k, v element.
template <int Dk, int ES>
struct BwdSmem {
  static constexpr int PER_THREAD = Dk / 4;           // state entries per thread
  static constexpr int TK = 0;                        // k        [kBlk][Dk]
  static constexpr int TA = TK + kBlk * Dk;           // alpha    [kBlk][Dk]
  static constexpr int TQ = TA + kBlk * Dk;           // q        [kBlk][Dk]
  static constexpr int TV = TQ + kBlk * Dk;           // v slice  [kBlk][32]
  static constexpr int TD = TV + kBlk * kCols;        // do slice [kBlk][32]
  static constexpr int TB = TD + kBlk * kCols;        // beta     [kBlk] (padded to 4)
  static constexpr int PY = TB + 4;                   // y parts  [2][4][32]
  static constexpr int PD = PY + 2 * 4 * kCols;       // du parts [2][4][32]
  static constexpr int ST = PD + 2 * 4 * kCols;       // states   [kBlk-2][PER_THREAD][128]
  // staging of the next block's tokens as they sit in global memory (bytes):
  // k, q [kBlk][Dk] x ES; g [kBlk][Dk] x 4; v slice [kBlk][32] x ES;
  // do slice [kBlk][32] x 4; beta [kBlk] x 4
  static constexpr int SK = 0, SQ = SK + kBlk * Dk * ES, SG = SQ + kBlk * Dk * ES;
  static constexpr int SV = SG + kBlk * Dk * 4, SD = SV + kBlk * kCols * ES;
  static constexpr int SB = SD + kBlk * kCols * 4, S_BYTES = SB + 16;
  static constexpr int STAGE = ST + (kBlk - 2) * PER_THREAD * kBThreads;
  static constexpr int TOTAL = STAGE + S_BYTES / 4;
};

// Thread layout: warp w owns rows [w Dk/4, (w+1) Dk/4) of the slice; lane
// (rg, cg) = (lane >> 3, lane & 7) owns the RT = Dk/16 rows starting at
// w Dk/4 + rg RT and the 4 columns starting at 4 cg.  Column sums over a
// warp's rows reduce-scatter across rg (lane bits 16, 8), row sums over the
// slice's columns across cg (lane bits 4, 2, 1).
template <typename TIn, int Dk, int Dv>
__global__ void __launch_bounds__(kBThreads, 4) backward_kernel(const BwdArgs a) {
  using L = BwdSmem<Dk, (int)sizeof(TIn)>;
  constexpr int RPW = Dk / 4, RT = Dk / 16, NS = Dv / kCols, DD = Dk * Dv;
  constexpr int RSH = 3 - Log2<RT>::value;   // row sums: lanes sharing a row differ in cg's low RSH bits
  extern __shared__ __align__(16) float smem[];
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int cg = lane & 7, rg = lane >> 3;
  const int H = a.H;
  const int slice = blockIdx.x % NS, unit = blockIdx.x / NS, n = unit / H, h = unit % H;
  const int c4 = cg * 4;                       // first column of the thread within the slice
  const int col = slice * kCols + c4;          // ... within the head
  const int rbase = w * RPW + rg * RT;         // first row of the thread
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

  // the thread's tile of S and dS: per row, columns (0, 1) and (2, 3) as
  // pairs for the paired FP32 units
  float2 S[RT][2], dS[RT][2];
  int par = 0;

  char *stage = reinterpret_cast<char *>(smem + L::STAGE);
  // Start the copies of the tokens [t_lo, t_lo + cnt) into the staging area
  // (q and do only when full); they land while the current block computes.
  auto issue_tokens = [&](int64_t t_lo, int cnt, bool full) {
    constexpr int KCH = Dk * (int)sizeof(TIn) / 16, GCH = Dk * 4 / 16;
    constexpr int VCH = kCols * (int)sizeof(TIn) / 16, DCH = kCols * 4 / 16;
    const size_t th0 = (size_t)(t_begin + t_lo) * H + h;   // (token, head) row of t_lo
    for (int e = tid; e < cnt * KCH; e += kBThreads) {
      const int s = e / KCH, x = e - s * KCH;
      const size_t off = ((th0 + (size_t)s * H) * Dk) * sizeof(TIn) + (size_t)x * 16;
      cp_async16(stage + L::SK + e * 16, reinterpret_cast<const char *>(a.k) + off);
      if (full) cp_async16(stage + L::SQ + e * 16, reinterpret_cast<const char *>(a.q) + off);
    }
    for (int e = tid; e < cnt * GCH; e += kBThreads) {
      const int s = e / GCH, x = e - s * GCH;
      cp_async16(stage + L::SG + e * 16,
                 reinterpret_cast<const char *>(a.g) + ((th0 + (size_t)s * H) * Dk) * 4 + (size_t)x * 16);
    }
    for (int e = tid; e < cnt * VCH; e += kBThreads) {
      const int s = e / VCH, x = e - s * VCH;
      cp_async16(stage + L::SV + e * 16,
                 reinterpret_cast<const char *>(a.v) +
                     ((th0 + (size_t)s * H) * Dv + slice * kCols) * sizeof(TIn) + (size_t)x * 16);
    }
    if (full)
      for (int e = tid; e < cnt * DCH; e += kBThreads) {
        const int s = e / DCH, x = e - s * DCH;
        cp_async16(stage + L::SD + e * 16,
                   reinterpret_cast<const char *>(a.dout) +
                       ((th0 + (size_t)s * H) * Dv + slice * kCols) * 4 + (size_t)x * 16);
      }
    if (tid < cnt) cp_async4(stage + L::SB + tid * 4, a.beta + th0 + (size_t)tid * H);
    cp_async_commit();
  };
  // Staged tokens -> FP32 token arrays (alpha = exp(g)).  Called between two
  // barriers, after every thread's copies have landed.
  auto unpack_tokens = [&](int cnt, bool full) {
    const TIn *sk = reinterpret_cast<const TIn *>(stage + L::SK);
    const TIn *sq = reinterpret_cast<const TIn *>(stage + L::SQ);
    const float *sg = reinterpret_cast<const float *>(stage + L::SG);
    for (int e = tid; e < cnt * Dk; e += kBThreads) {
      tk[e] = to_f32(sk[e]);
      ta[e] = __expf(sg[e]);
      if (full) tq[e] = to_f32(sq[e]);
    }
    const TIn *sv = reinterpret_cast<const TIn *>(stage + L::SV);
    const float *sd = reinterpret_cast<const float *>(stage + L::SD);
    for (int e = tid; e < cnt * kCols; e += kBThreads) {
      tv[e] = to_f32(sv[e]);
      if (full) tdo[e] = sd[e];
    }
    if (tid < cnt) tb[tid] = reinterpret_cast<const float *>(stage + L::SB)[tid];
  };
  // L2 prefetch of a stored state's slice: one 128-byte line per row.
  auto prefetch_state = [&](int64_t b) {
    if (tid < Dk) prefetch_l2(ck + (size_t)b * DD + (size_t)tid * Dv + slice * kCols);
  };
  // a [Dk][Dv] FP32 matrix in global memory <-> the thread's tile
  auto ld_tile = [&](const float *src, float2 (&X)[RT][2]) {
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const float4 x = *reinterpret_cast<const float4 *>(src + (size_t)(rbase + r) * Dv + col);
      X[r][0] = make_float2(x.x, x.y);
      X[r][1] = make_float2(x.z, x.w);
    }
  };
  auto st_tile = [&](float *dst, const float2 (&X)[RT][2]) {
#pragma unroll
    for (int r = 0; r < RT; ++r)
      *reinterpret_cast<float4 *>(dst + (size_t)(rbase + r) * Dv + col) =
          make_float4(X[r][0].x, X[r][0].y, X[r][1].x, X[r][1].y);
  };
  // The 4 columns' sums over all Dk rows of a per-thread part p (one value
  // per column): reduce-scatter over the warp's row groups, then the four
  // warps' parts meet in buf.
  auto col_sums_post = [&](const float2 (&p)[2], float *buf) {
    float v[4] = {p[0].x, p[0].y, p[1].x, p[1].y};
    buf[w * kCols + c4 + rg] = reduce_scatter<4, 16, 8>(v, lane);
  };
  auto col_sums_read = [&](const float *buf, float (&o)[4]) {
    float x0[4], x1[4], x2[4], x3[4];
    lds4(buf + c4, x0);
    lds4(buf + kCols + c4, x1);
    lds4(buf + 2 * kCols + c4, x2);
    lds4(buf + 3 * kCols + c4, x3);
#pragma unroll
    for (int c = 0; c < 4; ++c) o[c] = (x0[c] + x1[c]) + (x2[c] + x3[c]);
  };
  // One forward step of token slot s: S <- Diag(alpha) S + k u^T, with
  // y_j = sum_c alpha_c k_c S_cj and u = beta (v - y).
  auto fwd_step = [&](int s) {
    float kr[RT], ar[RT], vv[4];
    lds_rows<RT>(tk + s * Dk + rbase, kr);
    lds_rows<RT>(ta + s * Dk + rbase, ar);
    float2 yp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const float ak = ar[r] * kr[r];
      const float2 ak2 = make_float2(ak, ak);
      yp[0] = __ffma2_rn(ak2, S[r][0], yp[0]);
      yp[1] = __ffma2_rn(ak2, S[r][1], yp[1]);
    }
    float *pp = py + par * 4 * kCols;
    col_sums_post(yp, pp);
    __syncthreads();
    float y[4];
    col_sums_read(pp, y);
    par ^= 1;
    lds4(tv + s * kCols + c4, vv);
    const float bt = tb[s];
    const float2 u[2] = {make_float2(bt * (vv[0] - y[0]), bt * (vv[1] - y[1])),
                         make_float2(bt * (vv[2] - y[2]), bt * (vv[3] - y[3]))};
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const float2 a2 = make_float2(ar[r], ar[r]), k2 = make_float2(kr[r], kr[r]);
      S[r][0] = __ffma2_rn(a2, S[r][0], __fmul2_rn(k2, u[0]));
      S[r][1] = __ffma2_rn(a2, S[r][1], __fmul2_rn(k2, u[1]));
    }
  };
  // sum over the thread's 4 columns of X[r][.] * Y[.], for every row r
  auto row_dots = [&](const float2 (&X)[RT][2], const float2 (&Y)[2], float (&o)[RT]) {
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const float2 t = __ffma2_rn(X[r][1], Y[1], __fmul2_rn(X[r][0], Y[0]));
      o[r] = t.x + t.y;
    }
  };
  // Backward step of token slot s (token t): S holds S_{t-1}, dS the gradient
  // w.r.t. S_t from later tokens.
  auto bwd_step = [&](int s, int64_t t) {
    float kr[RT], ar[RT], qr[RT], dov4[4], vv[4];
    lds_rows<RT>(tk + s * Dk + rbase, kr);
    lds_rows<RT>(ta + s * Dk + rbase, ar);
    lds_rows<RT>(tq + s * Dk + rbase, qr);
    lds4(tdo + s * kCols + c4, dov4);
    const float2 dov[2] = {make_float2(dov4[0], dov4[1]), make_float2(dov4[2], dov4[3])};
    float2 yp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)}, dp[2] = {yp[0], yp[0]};
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const float ak = ar[r] * kr[r];
      const float2 ak2 = make_float2(ak, ak), q2 = make_float2(qr[r], qr[r]);
      const float2 k2 = make_float2(kr[r], kr[r]);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        yp[h2] = __ffma2_rn(ak2, S[r][h2], yp[h2]);
        dS[r][h2] = __ffma2_rn(q2, dov[h2], dS[r][h2]);
        dp[h2] = __ffma2_rn(k2, dS[r][h2], dp[h2]);
      }
    }
    float *pp = py + par * 4 * kCols, *pq = pdu + par * 4 * kCols;
    col_sums_post(yp, pp);
    col_sums_post(dp, pq);
    __syncthreads();
    float y[4], du4[4];
    col_sums_read(pp, y);
    col_sums_read(pq, du4);
    par ^= 1;
    lds4(tv + s * kCols + c4, vv);
    const float bt = tb[s];
    const float2 u[2] = {make_float2(bt * (vv[0] - y[0]), bt * (vv[1] - y[1])),
                         make_float2(bt * (vv[2] - y[2]), bt * (vv[3] - y[3]))};
    const float2 du[2] = {make_float2(du4[0], du4[1]), make_float2(du4[2], du4[3])};
    const size_t th = (size_t)(t_begin + t) * H + h;
    if (w == 0 && rg == 0)
      *reinterpret_cast<float4 *>(a.dv + th * Dv + col) =
          make_float4(bt * du4[0], bt * du4[1], bt * du4[2], bt * du4[3]);
    // this slice's parts of du.(v - y) and u.do: the 4 columns, then across cg
    const float u4[4] = {u[0].x, u[0].y, u[1].x, u[1].y};
    float db = 0.f, ud = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      db = fmaf(du4[c], vv[c] - y[c], db);
      ud = fmaf(u4[c], dov4[c], ud);
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
      db += __shfl_xor_sync(kFull, db, o);
      ud += __shfl_xor_sync(kFull, ud, o);
    }
    if (tid == 0) ob[th] = db;
    // row sums over the slice: r1 = S do, r3 = S du, r2 = dS u, r4 = sum_j dS_cj S_cj
    float tmp[RT];
    row_dots(S, dov, tmp);
    const float r1 = reduce_scatter<RT, 4, 1>(tmp, lane);
    row_dots(S, du, tmp);
    const float r3 = reduce_scatter<RT, 4, 1>(tmp, lane);
    row_dots(dS, u, tmp);
    const float r2 = reduce_scatter<RT, 4, 1>(tmp, lane);
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const float2 x = __ffma2_rn(dS[r][1], S[r][1], __fmul2_rn(dS[r][0], S[r][0]));
      tmp[r] = x.x + x.y;
    }
    const float r4 = reduce_scatter<RT, 4, 1>(tmp, lane);
    if ((cg & ((1 << RSH) - 1)) == 0) {
      const int c = rbase + (cg >> RSH);
      const float al = ta[s * Dk + c], kc = tk[s * Dk + c];
      const size_t o = th * Dk + c;
      // S_t = Diag(alpha) S_{t-1} + k u^T, so S_t do = alpha (S_{t-1} do) + k (u . do)
      oq[o] = fmaf(al, r1, kc * ud);
      okk[o] = r2 - bt * al * r3;
      og[o] = al * (r4 - bt * kc * r3);
    }
    // dS <- Diag(alpha) (dS - beta k du^T); k and alpha read again rather
    // than held through the row sums, which keeps the step within 128 registers
    lds_rows<RT>(tk + s * Dk + rbase, kr);
    lds_rows<RT>(ta + s * Dk + rbase, ar);
    const float2 nbd[2] = {make_float2(-bt * du4[0], -bt * du4[1]),
                           make_float2(-bt * du4[2], -bt * du4[3])};
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const float2 a2 = make_float2(ar[r], ar[r]), k2 = make_float2(kr[r], kr[r]);
      dS[r][0] = __fmul2_rn(a2, __ffma2_rn(k2, nbd[0], dS[r][0]));
      dS[r][1] = __fmul2_rn(a2, __ffma2_rn(k2, nbd[1], dS[r][1]));
    }
  };
  auto st_slot = [&](int slot) {
    float *p = st + (size_t)slot * RPW * kBThreads;
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      p[(r * 4 + 0) * kBThreads + tid] = S[r][0].x;
      p[(r * 4 + 1) * kBThreads + tid] = S[r][0].y;
      p[(r * 4 + 2) * kBThreads + tid] = S[r][1].x;
      p[(r * 4 + 3) * kBThreads + tid] = S[r][1].y;
    }
  };
  auto ld_slot = [&](int slot) {
    const float *p = st + (size_t)slot * RPW * kBThreads;
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      S[r][0] = make_float2(p[(r * 4 + 0) * kBThreads + tid], p[(r * 4 + 1) * kBThreads + tid]);
      S[r][1] = make_float2(p[(r * 4 + 2) * kBThreads + tid], p[(r * 4 + 3) * kBThreads + tid]);
    }
  };

  // ---------------- forward sweep: the state at the start of every block ----------------
  if (a.init) {
    ld_tile(a.init + (size_t)unit * DD, S);
  } else {
#pragma unroll
    for (int r = 0; r < RT; ++r) S[r][0] = S[r][1] = make_float2(0.f, 0.f);
  }
  auto block_len = [&](int64_t b) { return (int)((T - b * kBlk) < kBlk ? (T - b * kBlk) : kBlk); };
  if (nb > 0) issue_tokens(0, block_len(0), false);
  for (int64_t b = 0; b < nb; ++b) {
    const int cnt = block_len(b);
    st_tile(ck + (size_t)b * DD, S);
    cp_async_wait_all();
    __syncthreads();   // staged tokens visible; the previous block's tokens no longer read
    unpack_tokens(cnt, false);
    __syncthreads();   // tokens visible; staging free
    if (b + 1 < nb) issue_tokens((b + 1) * kBlk, block_len(b + 1), false);
    if (cnt == kBlk) {
#pragma unroll
      for (int s = 0; s < kBlk; ++s) fwd_step(s);
    } else {
      for (int s = 0; s < cnt; ++s) fwd_step(s);
    }
  }

  // ---------------- reverse sweep ----------------
  if (a.dfin) {
    ld_tile(a.dfin + (size_t)unit * DD, dS);
  } else {
#pragma unroll
    for (int r = 0; r < RT; ++r) dS[r][0] = dS[r][1] = make_float2(0.f, 0.f);
  }
  if (nb > 0) {
    issue_tokens((nb - 1) * kBlk, block_len(nb - 1), true);
    prefetch_state(nb - 1);
  }
  for (int64_t b = nb - 1; b >= 0; --b) {
    const int64_t t_lo = b * kBlk;
    const int cnt = block_len(b);
    cp_async_wait_all();
    __syncthreads();
    unpack_tokens(cnt, true);
    __syncthreads();
    if (b > 0) {
      issue_tokens((b - 1) * kBlk, kBlk, true);
      prefetch_state(b - 1);
    }
    ld_tile(ck + (size_t)b * DD, S);
    // replay: S becomes the state before token slot cnt-1; the states before
    // slots 1 .. cnt-2 are kept in slots 0 .. cnt-3, each thread its own entries
    if (cnt == kBlk) {   // full block: token slots are compile-time constants
#pragma unroll
      for (int s = 0; s + 1 < kBlk; ++s) {
        fwd_step(s);
        if (s + 1 < kBlk - 1) st_slot(s);
      }
#pragma unroll
      for (int s = kBlk - 1; s >= 0; --s) {
        if (s < kBlk - 1) {
          if (s >= 1) ld_slot(s - 1);
          else ld_tile(ck + (size_t)b * DD, S);
        }
        bwd_step(s, t_lo + s);
      }
    } else {
      for (int s = 0; s + 1 < cnt; ++s) {
        fwd_step(s);
        if (s + 1 < cnt - 1) st_slot(s);
      }
      for (int s = cnt - 1; s >= 0; --s) {
        if (s < cnt - 1) {
          if (s >= 1) ld_slot(s - 1);
          else ld_tile(ck + (size_t)b * DD, S);
        }
        bwd_step(s, t_lo + s);
      }
    }
  }
  if (a.dinit) st_tile(a.dinit + (size_t)unit * DD, dS);
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

template <int ES>
static size_t backward_smem_bytes(int Dk) {
  switch (Dk) {
    case 32: return sizeof(float) * BwdSmem<32, ES>::TOTAL;
    case 64: return sizeof(float) * BwdSmem<64, ES>::TOTAL;
    default: return sizeof(float) * BwdSmem<128, ES>::TOTAL;
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
  const size_t smem = backward_smem_bytes<(int)sizeof(TIn)>(DK);
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
