// KDA multi-token decode on the 5th-generation tensor cores (sm_100a), for
// BF16 q/k/v with D_k = D_v = 128 and drafts of up to 16 tokens.
//
// A draft of C tokens of one (sequence, head) is one chunk of the chunked
// form ("LLM - Semianalysis, Kimi K3 아키텍처", Methods 1, FlashKDA;
// "MoonshotAI/Kimi-K3 딥다이브", section 4-1).  With Gam_t = sum_{s<=t} g_s
// counted from the draft's first token and T = (I + L)^-1 Diag(beta),
// L_ts = beta_t sum_c k_tc k_sc exp(Gam_tc - Gam_sc) for s < t:
//
//   W = T Ktilde,  U = T V,  Ktilde_t = exp(Gam_t) k_t,  Qtilde_t = exp(Gam_t) q_t
//   V_new = U - W S0
//   o_t   = (Qtilde S0)_t + sum_{s<=t} P_ts V_new_s,  P_ts = sum_c q_tc k_sc exp(Gam_tc - Gam_sc)
//   S_a   = Diag(exp(Gam_a)) S0 + Khat^T V_new,  Khat_s = exp(Gam_a - Gam_s) k_s (s <= a, else 0)
//
// where a + 1 is the number of accepted tokens.  The recurrence needs 3 C D^2
// FP32 multiply-adds per (sequence, head) on the CUDA cores; here the two
// products with D^2 operands run on the tensor cores and only the C x C
// intra-draft part runs on the CUDA cores:
//   acc1 [v][n] = S0^T [W; Qtilde]^T       (M = 128 value columns, N = 32, K = 128)
//   acc2 [v][k] = exp(Gam_a) S0^T + V_new^T Khat   (M = 128, N = 128, K = 16)
// Both accumulators are FP32 in tensor memory, transposed (lane = value
// column v), so a warp's shared-memory accesses to the row-major FP32 state
// cover 128 consecutive bytes.  S0 is rounded to BF16 only as the operand of
// the first product, as in the two-pass prefill; the state itself is updated
// in FP32.
//
// The kernel is persistent, two CTAs of 256 threads per SM, so that one
// CTA's barriers and tensor-core round trips overlap the other's work.  Each
// unit's FP32 state comes in by one 64 KB bulk copy, whose buffer then holds
// the BF16 operand S0^T; the next unit's copy starts once the first product
// has read it.  The next unit's q, k, v and g rows (four tensor copies) land
// while the current unit runs its products.
#include <cuda.h>

#include "kda_common.cuh"
#include "kda_tc_util.cuh"
#include "kda_tma.cuh"

namespace kda {
namespace {

constexpr int kMD = 128;          // D_k = D_v
constexpr int kMC = 16;           // operand rows of the second product (tokens, padded)
constexpr int kMThreads = 256;

struct MtcLayout {
  static constexpr uint32_t SF = 0;              // float [128][128] FP32 state in (bulk copy), then
  static constexpr uint32_t AT = 0;              // S0^T, K-major A: rows v, columns k (2 blocks)
  static constexpr uint32_t B1 = 65536;          // [W; Qtilde], K-major B: rows n, columns k
  static constexpr uint32_t A2 = B1 + 8192;      // V_new, MN-major A: rows t, columns v
  static constexpr uint32_t B2 = A2 + 4096;      // Khat, MN-major B: rows t, columns k
  static constexpr uint32_t RQ = B2 + 4096;      // bf16 [16][128] q rows
  static constexpr uint32_t RK = RQ + 4096;      // bf16 [16][128] k rows
  static constexpr uint32_t RV = RK + 4096;      // bf16 [16][128] v rows
  static constexpr uint32_t RG = RV + 4096;      // float [16][128] g rows, then Gam in place
  static constexpr uint32_t RB = RG + 8192;      // float [16] beta
  static constexpr uint32_t UP = RB + 128;       // bf16 [16][128] U = T V
  static constexpr uint32_t LM = UP + 4096;      // float [16][16] L (strictly lower)
  static constexpr uint32_t PM = LM + 1024;      // float [16][16] P (lower, diagonal included)
  static constexpr uint32_t TM = PM + 1024;      // float [16][16] T
  static constexpr uint32_t DD = TM + 1024;      // float [128] exp(Gam_a)
  static constexpr uint32_t BAR = DD + 512;      // mbarriers: state in, raw rows, product 1, product 2
  static constexpr uint32_t TMEM_SLOT = BAR + 32;
  static constexpr uint32_t TOTAL = TMEM_SLOT + 8;
  static_assert(AT % 1024 == 0 && B1 % 1024 == 0 && A2 % 1024 == 0 && B2 % 1024 == 0, "tiles");
  static_assert(RQ % 128 == 0 && RG % 128 == 0 && BAR % 8 == 0, "alignment");
};

// Tensor maps of q, k, v and g as [tokens][H][128] with a box of one head's
// rows of one draft.
struct MtcMaps {
  CUtensorMap q, k, v, g;
};
constexpr uint32_t kAcc2 = 0;     // TMEM columns [0, 128): the state, transposed
constexpr uint32_t kAcc1 = 128;   // TMEM columns [128, 160): S0^T [W; Qtilde]^T

__device__ __forceinline__ float4 ld4_bf16(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// One BF16 value at (row, col) of a row tile with `rows` rows.
__device__ __forceinline__ void st_tile_bf16(uint8_t *tile, int rows, int row, int col, float x) {
  *reinterpret_cast<__nv_bfloat16 *>(tile + tc::tile_offset(rows, row, col >> 3) + 2 * (col & 7)) =
      __float2bfloat16_rn(x);
}

// MC: the operand rows this instance is built for (8 or 16); CT: the draft
// length when fixed at compile time (1..MC), so that the per-token guards fold
// away, or 0 for a length given at run time (at most MC).
template <int MC, int CT>
__global__ void __launch_bounds__(kMThreads, 2)
decode_multi_tc_kernel(const __grid_constant__ MtcMaps maps, const float *__restrict__ beta,
                       float *__restrict__ state,
                       __nv_bfloat16 *__restrict__ out, const int32_t *__restrict__ accept_len,
                       int C_arg, int H, int64_t units, int32_t *dev_status, uint64_t wait_ns) {
  using Lay = MtcLayout;
  static_assert(CT >= 0 && CT <= MC, "draft length");
  const int C = CT > 0 ? CT : C_arg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t *sp = smem_raw + (sb - sraw);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sp + Lay::BAR);
  float *gam = reinterpret_cast<float *>(sp + Lay::RG);
  float *s_beta = reinterpret_cast<float *>(sp + Lay::RB);
  float *s_L = reinterpret_cast<float *>(sp + Lay::LM);
  float *s_P = reinterpret_cast<float *>(sp + Lay::PM);
  float *s_T = reinterpret_cast<float *>(sp + Lay::TM);
  float *s_d = reinterpret_cast<float *>(sp + Lay::DD);
  const __nv_bfloat16 *rq = reinterpret_cast<const __nv_bfloat16 *>(sp + Lay::RQ);
  const __nv_bfloat16 *rk = reinterpret_cast<const __nv_bfloat16 *>(sp + Lay::RK);
  const __nv_bfloat16 *rv = reinterpret_cast<const __nv_bfloat16 *>(sp + Lay::RV);
  __nv_bfloat16 *s_up = reinterpret_cast<__nv_bfloat16 *>(sp + Lay::UP);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hw = warp >> 2;
  const int vrow = 32 * qd + lane;   // this thread's TMEM lane = value column
  int64_t u = blockIdx.x;
  if (u >= units) return;
  const int64_t G = gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.q)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.g)) : "memory");
  }
  if (warp == 0) tc::tmem_alloc(sb + Lay::TMEM_SLOT, 256);
  // Operand rows of tokens C..15 stay zero for the whole call.
  for (int i = tid; i < (8192 + 4096 + 4096) / 16; i += kMThreads)
    *reinterpret_cast<uint4 *>(sp + Lay::B1 + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + Lay::TMEM_SLOT);
  const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);

  // Copies and products in flight, tracked identically by every thread
  // (uniform decisions): bit 0 = state in, 1 = raw rows, 2 and 3 = products.
  uint32_t pend = 0;
  auto load_state = [&](int64_t unit) {   // one bulk copy (tid 0)
    if (tid == 0) {
      mbar_expect_tx(sb + Lay::BAR, kMD * kMD * 4);
      bulk_load(sb + Lay::SF, state + (size_t)unit * kMD * kMD, kMD * kMD * 4, sb + Lay::BAR);
    }
    pend |= 1u;
  };
  auto load_raw = [&](int64_t unit) {     // four tensor copies (tid 0)
    if (tid == 0) {
      const int n = (int)(unit / H), h = (int)(unit % H), z = n * C;
      const uint32_t bar = sb + Lay::BAR + 8;
      mbar_expect_tx(bar, (uint32_t)C * (3 * 256 + 512));
      tma_load_3d(sb + Lay::RQ, &maps.q, 0, h, z, bar);
      tma_load_3d(sb + Lay::RK, &maps.k, 0, h, z, bar);
      tma_load_3d(sb + Lay::RV, &maps.v, 0, h, z, bar);
      tma_load_3d(sb + Lay::RG, &maps.g, 0, h, z, bar);
    }
    if (warp == 0) {   // beta: one 4-byte async copy per token (strided by H)
      const int n = (int)(unit / H), h = (int)(unit % H);
      if (lane < C) cp_async4(sb + Lay::RB + 4 * lane, beta + ((size_t)n * C + lane) * H + h, true);
      cp_async_commit();
    }
    pend |= 2u;
  };
  // accepted length of the unit's sequence, read one unit ahead
  auto accepted = [&](int64_t unit) {
    int acc = C;
    if (accept_len && unit < units) {
      acc = accept_len[unit / H];
      acc = acc < 0 ? 0 : (acc > C ? C : acc);
    }
    return acc;
  };
  load_state(u);
  load_raw(u);

  uint32_t sph = 0, rph = 0, m1ph = 0, m2ph = 0;
  bool aborted = false;
  int acc_next = accepted(u);
  for (; u < units; u += G) {
    const int n = (int)(u / H), h = (int)(u % H);
    const int a = acc_next - 1;   // the stored state follows token a (none when a < 0)
    acc_next = accepted(u + G);

    // ---- the unit's rows; Gam (in place), beta and exp(Gam_a) ----
    if (__syncthreads_or(!wait_timed(bars + 1, rph, wait_ns))) { aborted = true; break; }
    if (warp == 0) cp_async_wait_all();   // beta, published by the barrier below
    rph ^= 1;
    pend &= ~2u;
    if (tid < kMD) {
      float gv[MC];
#pragma unroll
      for (int t = 0; t < MC; ++t) gv[t] = t < C ? gam[t * kMD + tid] : 0.f;
      float run = 0.f, ga = 0.f;
#pragma unroll
      for (int t = 0; t < MC; ++t) {
        run += gv[t];
        gv[t] = run;
        if (t == a) ga = run;
      }
#pragma unroll
      for (int t = 0; t < MC; ++t)
        if (t < C) gam[t * kMD + tid] = gv[t];
      s_d[tid] = a >= 0 ? __expf(ga) : 1.f;
    }
    __syncthreads();

    // ---- gated Gram products L (s < t) and P (s <= t): 4 lanes per pair, 64
    //      pairs per pass (one pass up to 8 tokens); group grp walks the 16-
    //      channel blocks in the order i ^ grp, so the 8 groups of a warp read 8
    //      different blocks of their rows at each step (no bank conflicts) ----
    {
      const int np = C * (C + 1) / 2, grp = lane >> 2, sub = lane & 3;
      for (int base = 0; base < np; base += 8 * (kMThreads / 32)) {
        const int p = base + 8 * warp + grp;
        const bool ok = p < np;
        int t = 0, s = 0;
        if (ok) {
          while ((t + 1) * (t + 2) / 2 <= p) ++t;
          s = p - t * (t + 1) / 2;
        }
        float kk = 0.f, qq = 0.f;
        if (ok) {
#pragma unroll 4
          for (int i = 0; i < 8; ++i) {
            const int c = 16 * (i ^ grp) + 4 * sub;
            const float4 gt = *reinterpret_cast<const float4 *>(gam + t * kMD + c);
            const float4 gs = *reinterpret_cast<const float4 *>(gam + s * kMD + c);
            const float4 kt = ld4_bf16(rk + t * kMD + c), ks = ld4_bf16(rk + s * kMD + c);
            const float4 qt = ld4_bf16(rq + t * kMD + c);
            // exp(Gam_t - Gam_s) <= 1 for s <= t: no overflow for any decay
            const float e0 = ks.x * __expf(gt.x - gs.x), e1 = ks.y * __expf(gt.y - gs.y);
            const float e2 = ks.z * __expf(gt.z - gs.z), e3 = ks.w * __expf(gt.w - gs.w);
            kk += kt.x * e0 + kt.y * e1 + kt.z * e2 + kt.w * e3;
            qq += qt.x * e0 + qt.y * e1 + qt.z * e2 + qt.w * e3;
          }
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
          kk += __shfl_xor_sync(0xffffffffu, kk, o);
          qq += __shfl_xor_sync(0xffffffffu, qq, o);
        }
        if (ok && sub == 0) {
          if (s < t) s_L[t * kMC + s] = s_beta[t] * kk;
          s_P[t * kMC + s] = qq;
        }
      }
    }
    __syncthreads();

    // ---- T = (I + L)^-1 Diag(beta) by forward substitution (warp 4, lane = column);
    //      meanwhile Qtilde and Khat (warps 0-3, one key channel per thread) ----
    float ktl[MC];   // Ktilde of this thread's channel (warps 0-3)
    if (warp == 4) {
      const int j = lane;
      float col[MC];
#pragma unroll
      for (int t = 0; t < MC; ++t) {
        float x = 0.f;
        if (t < C) {
          x = t == j ? s_beta[t] : 0.f;
#pragma unroll
          for (int s = 0; s < t; ++s) x -= s_L[t * kMC + s] * col[s];
        }
        col[t] = x;
      }
      if (j < MC)
#pragma unroll
        for (int t = 0; t < MC; ++t) s_T[t * kMC + j] = col[t];
    } else if (tid < kMD) {
      const int c = tid;
      const float ga = a >= 0 ? gam[a * kMD + c] : 0.f;
      float qt[MC], kh[MC];
#pragma unroll
      for (int t = 0; t < MC; ++t) {
        ktl[t] = qt[t] = kh[t] = 0.f;
        if (t < C) {
          const float G_t = gam[t * kMD + c];
          const float kv = __bfloat162float(rk[t * kMD + c]);
          const float eg = __expf(G_t);
          ktl[t] = kv * eg;
          qt[t] = __bfloat162float(rq[t * kMD + c]) * eg;
          kh[t] = t <= a ? kv * __expf(ga - G_t) : 0.f;
        }
      }
#pragma unroll
      for (int t = 0; t < MC; ++t)
        if (t < C) {
          st_tile_bf16(sp + Lay::B1, 2 * MC, MC + t, c, qt[t]);
          st_tile_bf16(sp + Lay::B2, 16, t, c, kh[t]);
        }
    }
    __syncthreads();

    // ---- W = T Ktilde (warps 0-3) and U = T V (warps 4-7) ----
    {
      const float *__restrict__ sT = s_T;
      const bool kside = tid < kMD;
      const int c = kside ? tid : tid - kMD;
      float src[MC];
#pragma unroll
      for (int s = 0; s < MC; ++s)
        src[s] = kside ? ktl[s] : (s < C ? __bfloat162float(rv[s * kMD + c]) : 0.f);
#pragma unroll
      for (int t = 0; t < MC; ++t) {
        if (t < C) {
          float x = 0.f;
#pragma unroll
          for (int s = 0; s <= t; ++s) x += sT[t * kMC + s] * src[s];
          if (kside) st_tile_bf16(sp + Lay::B1, 2 * MC, t, c, x);
          else s_up[t * kMD + c] = __float2bfloat16_rn(x);
        }
      }
    }
    tc::fence_smem_to_async();   // operand tiles for the products; raw rows refilled below

    // ---- S0 -> TMEM (scaled by exp(Gam_a)) and -> the BF16 operand S0^T, which
    //      takes the place of the FP32 rows once every thread has read its column ----
    if (__syncthreads_or(!wait_timed(bars + 0, sph, wait_ns))) { aborted = true; break; }
    sph ^= 1;
    pend &= ~1u;
    if (u + G < units) load_raw(u + G);   // every thread is past its last read of the rows
    {
      const float *sf = reinterpret_cast<const float *>(sp + Lay::SF);
      uint32_t pk[32];   // the thread's 64 values of S0 as BF16 pairs
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int k0 = 64 * hw + 16 * m;
        float x[16], y[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = sf[(k0 + e) * kMD + vrow];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 d4 = *reinterpret_cast<const float4 *>(s_d + k0 + e);
          y[e] = d4.x * x[e];
          y[e + 1] = d4.y * x[e + 1];
          y[e + 2] = d4.z * x[e + 2];
          y[e + 3] = d4.w * x[e + 3];
        }
        tc::tmem_st16(tl + kAcc2 + (uint32_t)k0, y);
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[8 * m + e] = tc::pack_bf16(x[2 * e], x[2 * e + 1]);
        asm volatile("" ::: "memory");   // one batch of loads at a time (registers)
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < 8; ++m)
        tc::st_shared_v4(sb + Lay::AT + tc::tile_offset(128, vrow, 8 * hw + m), pk[4 * m],
                         pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
      tc::tmem_wait_st();
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();

    // ---- acc1 = S0^T [W; Qtilde]^T ----
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id1 = tc::idesc_bf16(128, 2 * MC, 0, 0);
#pragma unroll
      for (int s = 0; s < kMD / 16; ++s)
        tc::mma_bf16(tmem + kAcc1, tc::desc_kmajor(sb + Lay::AT, 128, s),
                     tc::desc_kmajor(sb + Lay::B1, 2 * MC, s), id1, s > 0);
      tc::mma_commit(sb + Lay::BAR + 16);
    }
    pend |= 4u;
    if (__syncthreads_or(!wait_timed(bars + 2, m1ph, wait_ns))) { aborted = true; break; }
    m1ph ^= 1;
    pend &= ~4u;
    tc::fence_after_sync();
    if (u + G < units) load_state(u + G);   // the first product has read S0^T

    // ---- V_new = U - W S0 and the outputs (thread = value column; both warp
    //      halves form V_new, half hw writes the tokens of parity hw) ----
    {
      const float *__restrict__ sP = s_P;
      const __nv_bfloat16 *__restrict__ sU = s_up;
      float x[2 * MC];
      tc::tmem_ldw<2 * MC>(tl + kAcc1, x);
      tc::tmem_wait_ld();
      float vn[MC];
      __nv_bfloat16 *op = out + (((size_t)n * C) * H + h) * kMD + vrow;
#pragma unroll
      for (int t = 0; t < MC; ++t) {
        if (t < C) {
          vn[t] = __bfloat162float(sU[t * kMD + vrow]) - x[t];
          if ((t & 1) == hw) {
            float y = x[MC + t];
#pragma unroll
            for (int s = 0; s <= t; ++s) y += sP[t * kMC + s] * vn[s];
            op[(size_t)t * H * kMD] = __float2bfloat16_rn(y);
            st_tile_bf16(sp + Lay::A2, 16, t, vrow, vn[t]);
          }
        }
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();

    // ---- acc2 += V_new^T Khat; the state out (a warp writes 128 consecutive bytes) ----
    if (a >= 0) {
      if (tid == 0) {
        tc::fence_after_sync();
        tc::mma_bf16(tmem + kAcc2, tc::desc_mnmajor(sb + Lay::A2, 16, 0),
                     tc::desc_mnmajor(sb + Lay::B2, 16, 0), tc::idesc_bf16(128, 128, 1, 1), 1);
        tc::mma_commit(sb + Lay::BAR + 24);
      }
      pend |= 8u;
      if (__syncthreads_or(!wait_timed(bars + 3, m2ph, wait_ns))) { aborted = true; break; }
      m2ph ^= 1;
      pend &= ~8u;
      tc::fence_after_sync();
      float *so = state + (size_t)u * kMD * kMD + vrow;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int k0 = 64 * hw + 32 * m;
        float y[32];
        tc::tmem_ld32(tl + kAcc2 + (uint32_t)k0, y);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) __stcs(so + (size_t)(k0 + e) * kMD, y[e]);
      }
    }
    // No barrier here: the next unit's first wait is one, and every thread
    // reads (state out) and later writes (state in) the same TMEM columns.
    tc::fence_before_sync();
  }

  if (aborted) {
    report(dev_status, KDA_ERR_TIMEOUT);
    // copies and products still in flight end before the memory is released
    if (pend & 1u) wait_timed(bars + 0, sph, wait_ns);
    if (pend & 2u) wait_timed(bars + 1, rph, wait_ns);
    if (pend & 4u) wait_timed(bars + 2, m1ph, wait_ns);
    if (pend & 8u) wait_timed(bars + 3, m2ph, wait_ns);
  }
  cp_async_wait_all();   // beta's copies of a unit the loop did not reach
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool decode_multi_tc_supported(int dtype, int dk, int dv, int T_new) {
  return dtype == KDA_DTYPE_BF16 && dk == kMD && dv == kMD && T_new >= 1 && T_new <= kMC;
}

cudaError_t launch_decode_multi_tc(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float *state, void *out,
                                   const int32_t *accept_len, int T_new, int64_t units, int H,
                                   int32_t *dev_status, cudaStream_t stream) {
  if (units <= 0) return cudaSuccess;
  const int64_t tokens = units / H * T_new;
  MtcMaps maps;
  if (!make_map(&maps.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMD, H, tokens, kMD, T_new,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&maps.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMD, H, tokens, kMD, T_new,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&maps.v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kMD, H, tokens, kMD, T_new,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&maps.g, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kMD, H, tokens, kMD, T_new,
                CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  // One instance per draft length, so the per-token guards fold away: 0.523 ms
  // for 7 tokens through a run-time-length instance, against 0.423 for 8
  // through its own (512 x 32 heads).
  void (*kern)(MtcMaps, const float *, float *, __nv_bfloat16 *, const int32_t *, int, int,
               int64_t, int32_t *, uint64_t);
  switch (T_new) {
    case 1: kern = decode_multi_tc_kernel<8, 1>; break;
    case 2: kern = decode_multi_tc_kernel<8, 2>; break;
    case 3: kern = decode_multi_tc_kernel<8, 3>; break;
    case 4: kern = decode_multi_tc_kernel<8, 4>; break;
    case 5: kern = decode_multi_tc_kernel<8, 5>; break;
    case 6: kern = decode_multi_tc_kernel<8, 6>; break;
    case 7: kern = decode_multi_tc_kernel<8, 7>; break;
    case 8: kern = decode_multi_tc_kernel<8, 8>; break;
    case 9: kern = decode_multi_tc_kernel<16, 9>; break;
    case 10: kern = decode_multi_tc_kernel<16, 10>; break;
    case 11: kern = decode_multi_tc_kernel<16, 11>; break;
    case 12: kern = decode_multi_tc_kernel<16, 12>; break;
    case 13: kern = decode_multi_tc_kernel<16, 13>; break;
    case 14: kern = decode_multi_tc_kernel<16, 14>; break;
    case 15: kern = decode_multi_tc_kernel<16, 15>; break;
    default: kern = decode_multi_tc_kernel<16, 16>; break;
  }
  const size_t smem = MtcLayout::TOTAL + 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // two CTAs per SM need the whole shared-memory carveout
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, smem_sm = 0, reserved = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  // Two CTAs per SM when their shared memory fits (the registers are sized for
  // two by the launch bounds); the CTAs never wait on one another, so a grid
  // larger than what is resident is still correct.
  if (cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
    smem_sm = 0;
  if (cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    reserved = 1024;
  const int per_sm = (size_t)smem_sm >= 2 * (smem + (size_t)reserved) ? 2 : 1;
  const int64_t slots = (int64_t)per_sm * sms;
  const unsigned grid = (unsigned)(units < slots ? units : slots);
  kern<<<grid, kMThreads, smem, stream>>>(maps, beta, state, (__nv_bfloat16 *)out, accept_len,
                                          T_new, H, units, dev_status, 2000000000ull);
  return cudaGetLastError();
}

}  // namespace kda
