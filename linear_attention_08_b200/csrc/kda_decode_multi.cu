// KDA multi-token decode: T_new recurrent steps per (sequence, head) with the
// FP32 state held in registers across the draft (speculative-decoding
// verification).  The step is the decode step of "LLM - Semianalysis, Kimi K3
// 아키텍처" (charstring.tistory.com/2557), Methods 1 (FlashKDA), repeated:
//   y = A^T k, z = A^T q with A = Diag(alpha) S_{t-1};  u = beta (v - y);
//   S_t = A + k u^T;  o = z + (q . k) u.
#include "kda_common.cuh"
#include "kda_tma.cuh"

namespace kda {

// Multi-token decode (speculative-decoding verification): each (sequence,
// head) runs T_new tokens through the recurrence with its state held in
// registers, writes the output of every token, and stores the state reached
// after the first accept_len[n] tokens (all T_new when accept_len is null).
// One HBM round trip of the state serves all T_new tokens.
//
// The kernel is persistent: two CTAs per SM walk the (sequence, head) units,
// and while a CTA runs the token loop of one unit, the next unit's FP32 state
// (one bulk copy into shared memory, completing on an mbarrier) and the raw
// inputs of its first kMultiGroup tokens (16-byte async copies) are already on
// their way, so the SM's share of HBM bandwidth stays busy during the serial
// token loop.
//
// The recurrence is independent per value column, so each warp owns whole
// columns: lane (c, r) of warp w holds columns 16w + 4c .. 16w + 4c + 3 of
// state rows r*DK/8 .. (r+1)*DK/8 - 1, as (row 2i, row 2i+1) pairs for the
// paired FP32 units.  The sums over rows of y = A^T k and z = A^T q finish
// inside the warp (three shuffle rounds that halve the values a lane holds),
// so the token loop has no block barrier.
//
// Inside a group of kMultiGroup tokens the decay is applied lazily: with
// lam_j = prod_{i<=j} alpha_i (from the group start), the registers hold
// S'_j = S_j / lam_j, so token j reads y = S'^T (lam_j k), z = S'^T (lam_j q)
// and updates S' += (k / lam_j) u^T, one paired FMA per row pair, and the
// true state lam_j S'_j is formed only where it is stored or a group ends.
// lam_j is exp of the group's cumulative log-decay.  A group in which that
// leaves [-60, 60] for some channel (decays far steeper than the method's
// floor) would take k / lam_j out of FP32 range, so such a group runs exactly
// instead: the staged vectors are k, q, k and alpha_j, and every token decays
// the registers first (one vote per group decides, uniform over the block).
constexpr int kMultiGroup = 8;
constexpr float kMultiLogRange = 60.f;

// ROWS consecutive shared-memory floats: 16-byte loads (ROWS is a multiple of 4).
template <int ROWS>
__device__ __forceinline__ void load_rows(const float *src, float *dst) {
  static_assert(ROWS % 4 == 0, "whole float4s");
#pragma unroll
  for (int i = 0; i < ROWS; i += 4) {
    const float4 v = *reinterpret_cast<const float4 *>(src + i);
    dst[i] = v.x; dst[i + 1] = v.y; dst[i + 2] = v.z; dst[i + 3] = v.w;
  }
}

// Four consecutive values as floats (8- or 16-byte aligned).
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

template <int DK, int DV, typename TIn>
struct MultiLayout {
  static constexpr int G = kMultiGroup;
  static constexpr uint32_t STATE = 0;                                    // float [DK][DV]
  static constexpr uint32_t RAW_Q = DK * DV * 4;                          // TIn [G][DK]
  static constexpr uint32_t RAW_K = RAW_Q + G * DK * sizeof(TIn);         // TIn [G][DK]
  static constexpr uint32_t RAW_V = RAW_K + G * DK * sizeof(TIn);         // TIn [G][DV]
  static constexpr uint32_t RAW_G = RAW_V + G * DV * sizeof(TIn);         // float [G][DK]
  static constexpr uint32_t RAW_B = RAW_G + G * DK * 4;                   // float [G]
  static constexpr uint32_t BAR = RAW_B + 64;                             // mbarrier
  static constexpr uint32_t TOTAL = BAR + 16;
  static_assert(RAW_Q % 16 == 0 && RAW_G % 16 == 0 && BAR % 8 == 0, "alignment");
};

template <int DK, int DV, int THREADS, typename TIn>
__global__ void __launch_bounds__(THREADS, 2)
decode_multi_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                    const TIn *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, float *__restrict__ state,
                    TIn *__restrict__ out, const int32_t *__restrict__ accept_len, int T_new,
                    int H, int64_t units, int32_t *dev_status, uint64_t wait_ns) {
  using Lay = MultiLayout<DK, DV, TIn>;
  constexpr int V4 = DV / 4;
  constexpr int ROWS = DK / 8;        // eight row groups per warp
  constexpr int RP = ROWS / 2;        // row pairs per thread
  // Staged per-row vectors keep each row group's ROWS values at a padded
  // stride, so the eight distinct 16-byte loads of a warp hit distinct banks.
  constexpr int RS = ROWS % 8 == 0 ? ROWS + 4 : ROWS + 8;
  constexpr int DKP = 8 * RS;
  constexpr int G = kMultiGroup;
  static_assert(THREADS == 2 * DV && DV % 16 == 0 && ROWS % 4 == 0, "tile mismatch");

  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(16) float s_kl[G][DKP], s_ql[G][DKP], s_ki[G][DKP], s_lam[G][DKP];
  __shared__ float s_v[G][DV], s_beta[G], s_qk[G];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rgl = lane >> 2;               // row group
  const int cq = 4 * warp + (lane & 3);    // column quad
  const int r0 = rgl * ROWS;
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  // The thread's rows of the staged vectors and its column of v (token 0).
  const float *s_klr = &s_kl[0][rgl * RS], *s_qlr = &s_ql[0][rgl * RS];
  const float *s_kir = &s_ki[0][rgl * RS], *s_lr = &s_lam[0][rgl * RS];
  const float *s_vc = &s_v[0][4 * cq + (rgl & 3)];
  const uint32_t sb = smem_u32(smem_raw);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem_raw + Lay::BAR);
  int64_t u = blockIdx.x;
  if (u >= units) return;

  // Next unit's state: one bulk copy (tid 0); its first group's raw inputs:
  // 16-byte async copies spread over the block, beta by 4-byte copies.
  auto prefetch = [&](int64_t unit) {
    const int n = (int)(unit / H), h = (int)(unit % H);
    if (tid == 0) {
      mbar_expect_tx(sb + Lay::BAR, DK * DV * 4);
      bulk_load(sb + Lay::STATE, state + (size_t)unit * DK * DV, DK * DV * 4, sb + Lay::BAR);
    }
    constexpr int QCH = DK * (int)sizeof(TIn) / 16, VCH = DV * (int)sizeof(TIn) / 16;
    constexpr int GCH = DK * 4 / 16, PER = 2 * QCH + VCH + GCH;
    const int cnt = T_new < G ? T_new : G;
    for (int e = tid; e < cnt * PER; e += THREADS) {
      const int j = e / PER, r = e % PER;
      const size_t tok = ((size_t)n * T_new + j) * H + h;
      const uint8_t *src;
      uint32_t dst;
      if (r < QCH) {
        src = reinterpret_cast<const uint8_t *>(q + tok * DK) + 16 * r;
        dst = Lay::RAW_Q + j * DK * sizeof(TIn) + 16 * r;
      } else if (r < 2 * QCH) {
        src = reinterpret_cast<const uint8_t *>(k + tok * DK) + 16 * (r - QCH);
        dst = Lay::RAW_K + j * DK * sizeof(TIn) + 16 * (r - QCH);
      } else if (r < 2 * QCH + VCH) {
        src = reinterpret_cast<const uint8_t *>(v + tok * DV) + 16 * (r - 2 * QCH);
        dst = Lay::RAW_V + j * DV * sizeof(TIn) + 16 * (r - 2 * QCH);
      } else {
        src = reinterpret_cast<const uint8_t *>(g + tok * DK) + 16 * (r - 2 * QCH - VCH);
        dst = Lay::RAW_G + j * DK * 4 + 16 * (r - 2 * QCH - VCH);
      }
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sb + dst), "l"(src) : "memory");
    }
    if (tid < cnt) cp_async4(sb + Lay::RAW_B + 4 * tid, beta + ((size_t)n * T_new + tid) * H + h, true);
    cp_async_commit();
  };

  if (tid == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  prefetch(u);
  uint32_t phase = 0;
  bool aborted = false, exact = false;

  for (; u < units; u += gridDim.x) {
    const int n = (int)(u / H), h = (int)(u % H);
    int acc = T_new;
    if (accept_len) {
      acc = accept_len[n];
      acc = acc < 0 ? 0 : (acc > T_new ? T_new : acc);
    }
    if (__syncthreads_or(!wait_timed(bar, phase, wait_ns))) { aborted = true; break; }
    phase ^= 1;
    float2 sp[RP][4];   // sp[i][c] = (S[r0 + 2i][4cq + c], S[r0 + 2i + 1][4cq + c])
    {
      const float4 *S4s = reinterpret_cast<const float4 *>(smem_raw + Lay::STATE);
#pragma unroll
      for (int i = 0; i < RP; ++i) {
        const float4 x0 = S4s[(r0 + 2 * i) * V4 + cq];
        const float4 x1 = S4s[(r0 + 2 * i + 1) * V4 + cq];
        sp[i][0] = make_float2(x0.x, x1.x);
        sp[i][1] = make_float2(x0.y, x1.y);
        sp[i][2] = make_float2(x0.z, x1.z);
        sp[i][3] = make_float2(x0.w, x1.w);
      }
    }
    cp_async_wait_all();
    // Every thread has read the state and its token copies have landed: the
    // buffers may be refilled once the raw group is converted below.
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    float4 *S4 = reinterpret_cast<float4 *>(state + (size_t)u * DK * DV);

    for (int t0 = 0; t0 < T_new; t0 += G) {
      const int cnt = T_new - t0 < G ? T_new - t0 : G;
      // Stage the group, four consecutive channels per thread: lam k, lam q,
      // k / lam and lam from the cumulative log-decay since the group start
      // (or k, q, k and alpha in an exact group), and q . k (the QK lanes
      // holding one token reduce it by shuffles).  The
      // first group comes from the prefetched raw copies, later ones (drafts
      // longer than a group) straight from global memory.
      {
        constexpr int QK = DK / 4, QV = DV / 4;   // channel quads per token row
        static_assert(QK <= 32 && 32 % QK == 0, "a token's quads share one warp");
        const TIn *rq = reinterpret_cast<const TIn *>(smem_raw + Lay::RAW_Q);
        const TIn *rk = reinterpret_cast<const TIn *>(smem_raw + Lay::RAW_K);
        const TIn *rv = reinterpret_cast<const TIn *>(smem_raw + Lay::RAW_V);
        const float *rgp = reinterpret_cast<const float *>(smem_raw + Lay::RAW_G);
        const size_t tok0 = ((size_t)n * T_new + t0) * H + h;   // token (t0 + j): tok0 + j H
        // Cumulative log-decay of channels c..c+3 from the group start to token j.
        auto log_decay = [&](int j, int c) {
          float4 gs = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int i = 0; i <= j; ++i) {
            const float4 x = t0 == 0 ? load4(rgp + i * DK + c)
                                     : load4(g + (tok0 + (size_t)i * H) * DK + c);
            gs.x += x.x; gs.y += x.y; gs.z += x.z; gs.w += x.w;
          }
          return gs;
        };
        bool wide = false;
        for (int e = tid; e < cnt * QK; e += THREADS) {
          const float4 gs = log_decay(e / QK, 4 * (e % QK));
          const float lo = fminf(fminf(gs.x, gs.y), fminf(gs.z, gs.w));
          const float hi = fmaxf(fmaxf(gs.x, gs.y), fmaxf(gs.z, gs.w));
          wide |= !(lo >= -kMultiLogRange && hi <= kMultiLogRange);
        }
        exact = __syncthreads_or(wide);
        for (int base = warp * 32; base < cnt * QK; base += THREADS) {   // whole warps: shuffles below
          const int e = base + lane;
          const bool ok = e < cnt * QK;
          const int j = ok ? e / QK : 0, c = 4 * (e % QK);
          float4 kc, qc, lm, il;
          if (t0 == 0) {
            kc = load4(rk + j * DK + c);
            qc = load4(rq + j * DK + c);
          } else {
            const size_t off = (tok0 + (size_t)j * H) * DK + c;
            kc = load4(k + off);
            qc = load4(q + off);
          }
          if (!exact) {
            const float4 gs = log_decay(j, c);
            lm = make_float4(__expf(gs.x), __expf(gs.y), __expf(gs.z), __expf(gs.w));
            il = make_float4(__expf(-gs.x), __expf(-gs.y), __expf(-gs.z), __expf(-gs.w));
          } else {   // k, q, k and the token's own decay
            const float4 gj = t0 == 0 ? load4(rgp + j * DK + c) : load4(g + (tok0 + (size_t)j * H) * DK + c);
            lm = make_float4(__expf(gj.x), __expf(gj.y), __expf(gj.z), __expf(gj.w));
            il = make_float4(1.f, 1.f, 1.f, 1.f);
          }
          const float4 ls = exact ? il : lm;   // the scale of k and q
          float qk = qc.x * kc.x + qc.y * kc.y + qc.z * kc.z + qc.w * kc.w;
#pragma unroll
          for (int o = QK / 2; o > 0; o >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, o);
          if (ok) {
            const int pc = (c / ROWS) * RS + c % ROWS;
            *reinterpret_cast<float4 *>(&s_kl[j][pc]) = make_float4(ls.x * kc.x, ls.y * kc.y, ls.z * kc.z, ls.w * kc.w);
            *reinterpret_cast<float4 *>(&s_ql[j][pc]) = make_float4(ls.x * qc.x, ls.y * qc.y, ls.z * qc.z, ls.w * qc.w);
            *reinterpret_cast<float4 *>(&s_ki[j][pc]) = make_float4(il.x * kc.x, il.y * kc.y, il.z * kc.z, il.w * kc.w);
            *reinterpret_cast<float4 *>(&s_lam[j][pc]) = lm;
            if (c == 0) s_qk[j] = qk;
          }
        }
        for (int e = tid; e < cnt * QV; e += THREADS) {
          const int j = e / QV, c = 4 * (e % QV);
          *reinterpret_cast<float4 *>(&s_v[j][c]) =
              t0 == 0 ? load4(rv + j * DV + c) : load4(v + (tok0 + (size_t)j * H) * DV + c);
        }
        if (tid < cnt)
          s_beta[tid] = t0 == 0 ? reinterpret_cast<const float *>(smem_raw + Lay::RAW_B)[tid]
                                : beta[tok0 + (size_t)tid * H];
        __syncthreads();
        if (t0 == 0) {
          const int64_t nx = u + gridDim.x;   // the raw and state buffers are free now
          if (nx < units) prefetch(nx);
        }
      }

      // The group's tokens.  An exact group decays the registers by alpha_j
      // before each token.
      const int js = acc - 1 - t0;   // the accepted state is stored after token js
      TIn *op = out + (((size_t)n * T_new + t0) * H + h) * DV + 4 * cq + (rgl & 3);
      const size_t ostep = (size_t)H * DV;
#pragma unroll 1
      for (int j = 0; j < cnt; ++j) {
        if (exact) {   // A = Diag(alpha_j) S_{t-1} in the registers, four rows at a time
#pragma unroll
          for (int i = 0; i < RP; i += 2) {
            const float4 a = *reinterpret_cast<const float4 *>(s_lr + j * DKP + 2 * i);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              sp[i][c] = __fmul2_rn(make_float2(a.x, a.y), sp[i][c]);
              sp[i + 1][c] = __fmul2_rn(make_float2(a.z, a.w), sp[i + 1][c]);
            }
          }
        }
        float2 yp[4], zp[4];   // (even rows, odd rows) partial sums per column
        {
          float kl[ROWS], ql[ROWS];
          load_rows<ROWS>(s_klr + j * DKP, kl);
          load_rows<ROWS>(s_qlr + j * DKP, ql);
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            const float2 ka = make_float2(kl[2 * i], kl[2 * i + 1]);
            const float2 qa = make_float2(ql[2 * i], ql[2 * i + 1]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              yp[c] = i == 0 ? __fmul2_rn(ka, sp[0][c]) : __ffma2_rn(ka, sp[i][c], yp[c]);
              zp[c] = i == 0 ? __fmul2_rn(qa, sp[0][c]) : __ffma2_rn(qa, sp[i][c], zp[c]);
            }
          }
        }
        // Sum over the eight row groups (lane bits 2..4): each round sends half
        // of the values still held and keeps the other half, so lane (c, r)
        // ends with value r of (y_0..y_3, z_0..z_3) of its column quad.
        float r8[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) { r8[c] = yp[c].x + yp[c].y; r8[4 + c] = zp[c].x + zp[c].y; }
        float r4[4], r2[2];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float send = b4 ? r8[m] : r8[m + 4], keep = b4 ? r8[m + 4] : r8[m];
          r4[m] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const float send = b3 ? r4[m] : r4[m + 2], keep = b3 ? r4[m + 2] : r4[m];
          r2[m] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        const float r1 = (b2 ? r2[1] : r2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? r2[0] : r2[1], 4);
        const float uu = s_beta[j] * (s_vc[j * DV] - r1);          // the y lanes (r < 4)
        const float uz = __shfl_xor_sync(0xffffffffu, uu, 16);     // u beside each z lane
        if (rgl >= 4) op[j * ostep] = from_f32<TIn>(r1 + s_qk[j] * uz);
        float2 up[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float x = __shfl_sync(0xffffffffu, uu, (lane & 3) + 4 * m);
          up[m] = make_float2(x, x);
        }
        {
          float ki[ROWS];
          load_rows<ROWS>(s_kir + j * DKP, ki);
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            const float2 kc = make_float2(ki[2 * i], ki[2 * i + 1]);
#pragma unroll
            for (int c = 0; c < 4; ++c) sp[i][c] = __ffma2_rn(kc, up[c], sp[i][c]);
          }
        }
        if (j == js) {   // the state after the accepted tokens: lam_j S' (S itself when exact)
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            float a = 1.f, b = 1.f;
            if (!exact) {
              const float2 ab = *reinterpret_cast<const float2 *>(s_lr + j * DKP + 2 * i);
              a = ab.x;
              b = ab.y;
            }
            __stcs(&S4[(r0 + 2 * i) * V4 + cq],
                   make_float4(a * sp[i][0].x, a * sp[i][1].x, a * sp[i][2].x, a * sp[i][3].x));
            __stcs(&S4[(r0 + 2 * i + 1) * V4 + cq],
                   make_float4(b * sp[i][0].y, b * sp[i][1].y, b * sp[i][2].y, b * sp[i][3].y));
          }
        }
      }
      if (!exact && t0 + G < T_new) {   // the next group starts from the true state
        float lm[ROWS];
        load_rows<ROWS>(s_lr + (cnt - 1) * DKP, lm);
#pragma unroll
        for (int i = 0; i < RP; ++i) {
          const float2 a = make_float2(lm[2 * i], lm[2 * i + 1]);
#pragma unroll
          for (int c = 0; c < 4; ++c) sp[i][c] = __fmul2_rn(a, sp[i][c]);
        }
      }
      __syncthreads();   // the staged group is overwritten by the next one
    }
  }
  cp_async_wait_all();
  if (aborted) {
    report(dev_status, KDA_ERR_TIMEOUT);
    wait_timed(bar, phase, wait_ns);   // the state copy in flight, if any
  }
}

static int multi_num_sms() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    v = 148;
  return v;
}

template <int DK, int DV, typename TIn>
static cudaError_t launch_decode_multi_t(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta, float *state,
                                         void *out, const int32_t *accept_len, int T_new,
                                         int64_t units, int H, int32_t *dev_status,
                                         cudaStream_t stream) {
  // Two threads per value column: DV / 16 warps of 4 column quads x 8 row groups.
  constexpr int THREADS = 2 * DV;
  if (units <= 0) return cudaSuccess;
  auto kern = decode_multi_kernel<DK, DV, THREADS, TIn>;
  const size_t smem = MultiLayout<DK, DV, TIn>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int per_sm = 0;   // resident CTAs per SM (two at D_k = D_v = 128, more for smaller heads)
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, smem) != cudaSuccess ||
      per_sm <= 0)
    per_sm = 1;
  const int64_t slots = (int64_t)per_sm * multi_num_sms();
  const unsigned grid = (unsigned)(units < slots ? units : slots);
  kern<<<grid, THREADS, smem, stream>>>((const TIn *)q, (const TIn *)k, (const TIn *)v, g, beta,
                                        state, (TIn *)out, accept_len, T_new, H, units, dev_status,
                                        2000000000ull);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t launch_decode_multi_d(int dk, int dv, const void *q, const void *k,
                                         const void *v, const float *g, const float *beta,
                                         float *state, void *out, const int32_t *accept_len,
                                         int T_new, int64_t units, int H, int32_t *dev_status,
                                         cudaStream_t stream) {
#define KDA_DECM(DK_, DV_)                                                                  \
  if (dk == DK_ && dv == DV_)                                                               \
    return launch_decode_multi_t<DK_, DV_, TIn>(q, k, v, g, beta, state, out, accept_len,   \
                                                T_new, units, H, dev_status, stream);
  KDA_DECM(32, 32) KDA_DECM(32, 64) KDA_DECM(32, 128)
  KDA_DECM(64, 32) KDA_DECM(64, 64) KDA_DECM(64, 128)
  KDA_DECM(128, 32) KDA_DECM(128, 64) KDA_DECM(128, 128)
#undef KDA_DECM
  return cudaErrorInvalidValue;
}

// The tensor-core form (kda_decode_multi_tc.cu): BF16, D_k = D_v = 128, up to 16 tokens.
bool decode_multi_tc_supported(int dtype, int dk, int dv, int T_new);
cudaError_t launch_decode_multi_tc(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float *state, void *out,
                                   const int32_t *accept_len, int T_new, int64_t units, int H,
                                   int32_t *dev_status, cudaStream_t stream);

cudaError_t launch_decode_multi(int dtype, int dk, int dv, const void *q, const void *k,
                                const void *v, const float *g, const float *beta, float *state,
                                void *out, const int32_t *accept_len, int T_new, int64_t units,
                                int H, int32_t *dev_status, cudaStream_t stream) {
  if (decode_multi_tc_supported(dtype, dk, dv, T_new))
    return launch_decode_multi_tc(q, k, v, g, beta, state, out, accept_len, T_new, units, H,
                                  dev_status, stream);
  if (dtype == KDA_DTYPE_BF16)
    return launch_decode_multi_d<__nv_bfloat16>(dk, dv, q, k, v, g, beta, state, out,
                                                accept_len, T_new, units, H, dev_status, stream);
  return launch_decode_multi_d<float>(dk, dv, q, k, v, g, beta, state, out, accept_len, T_new,
                                      units, H, dev_status, stream);
}

}  // namespace kda
