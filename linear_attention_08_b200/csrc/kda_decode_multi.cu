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
// token loop.  Tokens are prepared in groups of kMultiGroup (gates and q . k
// for the whole group before the token loop), so each token costs two block
// barriers and no global-memory latency.  Each thread keeps four columns of a
// block of consecutive state rows, held as (row 2i, row 2i+1) pairs so that
// the paired FP32 instructions take a token's per-row gate values in pairs
// straight from 16-byte shared-memory loads.
constexpr int kMultiGroup = 8;

// ROWS consecutive shared-memory floats (the same for every lane of a warp):
// 16-byte loads when ROWS is a multiple of 4.
template <int ROWS>
__device__ __forceinline__ void load_rows(const float *src, float *dst) {
  if constexpr (ROWS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < ROWS; i += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + i);
      dst[i] = v.x; dst[i + 1] = v.y; dst[i + 2] = v.z; dst[i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < ROWS; ++i) dst[i] = src[i];
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
  constexpr int RPP = THREADS / V4;
  constexpr int ROWS = DK / RPP;
  constexpr int G = kMultiGroup;
  static_assert(THREADS % V4 == 0 && DK % RPP == 0 && ROWS % 2 == 0, "tile mismatch");
  constexpr int RP = ROWS / 2;   // row pairs per thread

  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(16) float s_ka[G][DK], s_qa[G][DK], s_alpha[G][DK], s_k[G][DK];
  __shared__ float s_v[G][DV], s_beta[G], s_qk[G];
  __shared__ float s_u[2][DV];
  __shared__ float4 s_red[2][2][RPP][V4];

  const int tid = threadIdx.x, cg = tid % V4, rg = tid / V4;
  const int lane = tid & 31, warp = tid >> 5;
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
  bool aborted = false;

  for (; u < units; u += gridDim.x) {
    const int n = (int)(u / H), h = (int)(u % H);
    int acc = T_new;
    if (accept_len) {
      acc = accept_len[n];
      acc = acc < 0 ? 0 : (acc > T_new ? T_new : acc);
    }
    if (__syncthreads_or(!wait_timed(bar, phase, wait_ns))) { aborted = true; break; }
    phase ^= 1;
    // The thread's four columns of each pair of consecutive rows, as
    // (row 2i, row 2i+1) pairs for the paired FP32 units: sp[i][c].
    float2 sp[RP][4];
    {
      const float4 *S4s = reinterpret_cast<const float4 *>(smem_raw + Lay::STATE);
#pragma unroll
      for (int i = 0; i < RP; ++i) {
        const float4 x0 = S4s[(rg * ROWS + 2 * i) * V4 + cg];
        const float4 x1 = S4s[(rg * ROWS + 2 * i + 1) * V4 + cg];
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
      // Stage the group: gates, alpha k, alpha q and q . k for every token at
      // once, four consecutive channels per thread (the QK lanes holding one
      // token reduce q . k by shuffles).  The first group comes from the
      // prefetched raw copies, later ones (drafts longer than a group)
      // straight from global memory.
      {
        constexpr int QK = DK / 4, QV = DV / 4;   // channel quads per token row
        static_assert(QK <= 32 && 32 % QK == 0, "a token's quads share one warp");
        const TIn *rq = reinterpret_cast<const TIn *>(smem_raw + Lay::RAW_Q);
        const TIn *rk = reinterpret_cast<const TIn *>(smem_raw + Lay::RAW_K);
        const TIn *rv = reinterpret_cast<const TIn *>(smem_raw + Lay::RAW_V);
        const float *rgp = reinterpret_cast<const float *>(smem_raw + Lay::RAW_G);
        const size_t tok0 = ((size_t)n * T_new + t0) * H + h;   // token (t0 + j): tok0 + j H
        for (int base = warp * 32; base < cnt * QK; base += THREADS) {   // whole warps: shuffles below
          const int e = base + lane;
          const bool ok = e < cnt * QK;
          const int j = ok ? e / QK : 0, c = 4 * (e % QK);
          float4 kc, qc, gc;
          if (t0 == 0) {
            kc = load4(rk + j * DK + c);
            qc = load4(rq + j * DK + c);
            gc = *reinterpret_cast<const float4 *>(rgp + j * DK + c);
          } else {
            const size_t off = (tok0 + (size_t)j * H) * DK + c;
            kc = load4(k + off);
            qc = load4(q + off);
            gc = *reinterpret_cast<const float4 *>(g + off);
          }
          const float4 al = make_float4(__expf(gc.x), __expf(gc.y), __expf(gc.z), __expf(gc.w));
          float qk = qc.x * kc.x + qc.y * kc.y + qc.z * kc.z + qc.w * kc.w;
#pragma unroll
          for (int o = QK / 2; o > 0; o >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, o);
          if (ok) {
            *reinterpret_cast<float4 *>(&s_alpha[j][c]) = al;
            *reinterpret_cast<float4 *>(&s_k[j][c]) = kc;
            *reinterpret_cast<float4 *>(&s_ka[j][c]) = make_float4(al.x * kc.x, al.y * kc.y, al.z * kc.z, al.w * kc.w);
            *reinterpret_cast<float4 *>(&s_qa[j][c]) = make_float4(al.x * qc.x, al.y * qc.y, al.z * qc.z, al.w * qc.w);
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

      for (int j = 0; j < cnt; ++j) {
        const int t = t0 + j, p = t & 1;   // parity-indexed buffers: no third barrier
        float kar[ROWS], qar[ROWS];
        load_rows<ROWS>(&s_ka[j][rg * ROWS], kar);
        load_rows<ROWS>(&s_qa[j][rg * ROWS], qar);
        float2 yp[4], zp[4];   // (even rows, odd rows) partial sums per column
#pragma unroll
        for (int c = 0; c < 4; ++c) yp[c] = zp[c] = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < RP; ++i) {
          const float2 ka = make_float2(kar[2 * i], kar[2 * i + 1]);
          const float2 qa = make_float2(qar[2 * i], qar[2 * i + 1]);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            yp[c] = __ffma2_rn(ka, sp[i][c], yp[c]);
            zp[c] = __ffma2_rn(qa, sp[i][c], zp[c]);
          }
        }
        s_red[p][0][rg][cg] = make_float4(yp[0].x + yp[0].y, yp[1].x + yp[1].y, yp[2].x + yp[2].y, yp[3].x + yp[3].y);
        s_red[p][1][rg][cg] = make_float4(zp[0].x + zp[0].y, zp[1].x + zp[1].y, zp[2].x + zp[2].y, zp[3].x + zp[3].y);
        __syncthreads();
        if (tid < DV) {
          const int c4 = tid >> 2, lane4 = tid & 3;
          float yy = 0.f, zz = 0.f;
#pragma unroll 8
          for (int r = 0; r < RPP; ++r) {
            yy += reinterpret_cast<const float *>(&s_red[p][0][r][c4])[lane4];
            zz += reinterpret_cast<const float *>(&s_red[p][1][r][c4])[lane4];
          }
          const float uu = s_beta[j] * (s_v[j][tid] - yy);
          s_u[p][tid] = uu;
          out[(((size_t)n * T_new + t) * H + h) * DV + tid] = from_f32<TIn>(zz + s_qk[j] * uu);
        }
        __syncthreads();
        const float4 u4 = reinterpret_cast<const float4 *>(s_u[p])[cg];
        const float2 uu[4] = {make_float2(u4.x, u4.x), make_float2(u4.y, u4.y),
                              make_float2(u4.z, u4.z), make_float2(u4.w, u4.w)};
        float alr[ROWS], kr[ROWS];
        load_rows<ROWS>(&s_alpha[j][rg * ROWS], alr);
        load_rows<ROWS>(&s_k[j][rg * ROWS], kr);
#pragma unroll
        for (int i = 0; i < RP; ++i) {
          const float2 a = make_float2(alr[2 * i], alr[2 * i + 1]);
          const float2 kc = make_float2(kr[2 * i], kr[2 * i + 1]);
#pragma unroll
          for (int c = 0; c < 4; ++c) sp[i][c] = __ffma2_rn(a, sp[i][c], __fmul2_rn(kc, uu[c]));
        }
        if (t + 1 == acc)
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            __stcs(&S4[(rg * ROWS + 2 * i) * V4 + cg], make_float4(sp[i][0].x, sp[i][1].x, sp[i][2].x, sp[i][3].x));
            __stcs(&S4[(rg * ROWS + 2 * i + 1) * V4 + cg], make_float4(sp[i][0].y, sp[i][1].y, sp[i][2].y, sp[i][3].y));
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
  // Two or more rows per thread (the row pairs of the paired FP32 units).
  constexpr int THREADS = (DK == 32 && DV == 32) ? 128 : 256;
  if (units <= 0) return cudaSuccess;
  auto kern = decode_multi_kernel<DK, DV, THREADS, TIn>;
  const size_t smem = MultiLayout<DK, DV, TIn>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t slots = 2 * (int64_t)multi_num_sms();
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

cudaError_t launch_decode_multi(int dtype, int dk, int dv, const void *q, const void *k,
                                const void *v, const float *g, const float *beta, float *state,
                                void *out, const int32_t *accept_len, int T_new, int64_t units,
                                int H, int32_t *dev_status, cudaStream_t stream) {
  if (dtype == KDA_DTYPE_BF16)
    return launch_decode_multi_d<__nv_bfloat16>(dk, dv, q, k, v, g, beta, state, out,
                                                accept_len, T_new, units, H, dev_status, stream);
  return launch_decode_multi_d<float>(dk, dv, q, k, v, g, beta, state, out, accept_len, T_new,
                                      units, H, dev_status, stream);
}

}  // namespace kda
