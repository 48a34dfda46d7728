// KDA chunked prefill on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Covers BF16 q/k/v/out with D_k = D_v = 128 and 64-token chunks; the FP32
// state never leaves the chip between chunks.  The method: prefill groups the
// tokens into chunks, unrolls the recurrence inside a chunk into dense matrix
// products and carries the state between chunks
// ("LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557),
// Methods 1, FlashKDA; "MoonshotAI/Kimi-K3 딥다이브" (fiv.co.kr/repos/kimi-k3-deep-dive.html),
// section 4-1, chunk-parallel tiles with a recurrence between them).
//
// One CTA owns one (sequence, head, slice of DVS value columns) and walks its
// sequence chunk by chunk.  For a chunk of 64 tokens starting from S0, with
// Gam_r = sum_{s<=r} g_s (inclusive, per channel):
//
//   M_ri = beta_r sum_c k_rc k_ic exp(Gam_rc - Gam_ic)   (i < r)  gated Gram of k
//   P_ri = sum_c q_rc k_ic exp(Gam_rc - Gam_ic)          (i <= r) gated q.k^T
//   T    = (I + M)^-1 diag(beta)                          UT transform
//   X    = V - Ktilde S0               (Ktilde_r = k_r exp(Gam_r))
//   U    = T X                                            delta-rule corrections
//   O    = Qtilde S0 + P U             (Qtilde_r = q_r exp(Gam_r))
//   S    = Diag(exp(Gam_63)) S0 + Khat^T U   (Khat_r = k_r exp(Gam_63 - Gam_r))
//
// Gate numerics: exp(Gam_r - Gam_i) is split into a factor on each operand
// so that both stay inside the FP32/BF16 exponent range.  With g >= -5 a
// factor exp(+-(Gam_r - ref)) is at most e^80 when the reference sits in the
// middle of a 32-token half, so each row r is scaled against the middle of
// its own half (Gam_15 or Gam_47).  The key operand then comes in two
// versions: k_i exp(Gam_15 - Gam_i) (i < 32) for rows of the first half and
// k_i exp(Gam_47 - Gam_i) (i < 64) for rows of the second; one MMA with
// N = 32 + 64 forms every needed product (the cross products are never
// read).  In the second version a factor for i < 32 can underflow; the
// product it belongs to is then below e^-12 (the other factor is at most
// e^75), far below the BF16 rounding of the operands.
//
// Tensor-core work per chunk (BF16 operands in 128-byte-swizzled shared
// tiles, FP32 accumulators in tensor memory):
//   Gram:   [k x; q x] (128x128) x [B^(0) | B^(1)] (96x128)^T -> M, P
//   MMA1:   [Ktilde; Qtilde] (128x128) x S0_bf16   -> Ktilde S0, Qtilde S0
//           (issued with the Gram product: it needs only the gates and S0)
//   MMA-U:  [T;P] (128x64) x X (64xDVS)            -> U (rows 0..63)
//   MMA2:   [T;P] x U accumulated onto MMA1 (rows 64..127 become O),
//           Khat^T (128x64) x U                     -> state increment
// The state-dependent chain per chunk is MMA1 -> X -> MMA-U -> MMA2.
// The triangular solve, the gates and the FP32 state update run on the SIMT
// pipes.  The FP32 state of the CTA's slice stays in registers: row c of the
// state belongs to TMEM lane c.
#include <cuda.h>

#include "kda_common.cuh"
#include "kda_tc_util.cuh"
#include "kda_tma.cuh"

namespace kda {
namespace {

constexpr int kC = 64;      // chunk length
constexpr int kDK = 128;    // key head size
constexpr int kDV = 128;    // value head size (full)
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kLd = 68;     // row stride of the FP32 64x64 scratch matrices (16-byte rows)

template <int DVS>
struct Layout {
  static constexpr uint32_t S_T = 0;                              // [128][DVS]  state, MN-major B
  static constexpr uint32_t WQ_T = S_T + 128 * DVS * 2;           // [128][128]  Ktilde;Qtilde, K-major A
  static constexpr uint32_t TP_T = WQ_T + 32768;                  // [128][64]   T;P, K-major A
  static constexpr uint32_t KH_T = TP_T + 16384;                  // [64][128]   Khat, MN-major A
  static constexpr uint32_t KV_T = KH_T + 16384;                  // [64][128+DVS]: X then U | V
  static constexpr uint32_t U_T = KV_T;                           // [64][DVS] X, then U, MN-major B
  static constexpr uint32_t G = KV_T + 64 * (128 + DVS) * 2;      // 72 KB region, used in turn for:
  static constexpr uint32_t STG_Q = G, STG_K = G + 16384;         //  next chunk's q, k [64][128] bf16
  static constexpr uint32_t STG_G = G + 32768;                    //  next chunk's g [64][128] fp32
  static constexpr uint32_t RED = G + 65536;                      //  float [8][128] scan partials
  static constexpr uint32_t GA = G;                               //  Gram A [128][128] K-major
  static constexpr uint32_t GB = G + 32768;                       //  Gram B [96][128] K-major
  static constexpr uint32_t MM = G;                               //  float [64][68] M
  static constexpr uint32_t XM = G + 17408;                       //  float [64][68] (I + M)^-1
  static constexpr uint32_t YS = G + 34816;                       //  float [2][16][17]
  static constexpr uint32_t ZS = G + 36992;                       //  float [32][36]
  static constexpr uint32_t MT = G + 41600;                       //  float [32][33] M_(1,0)^T
  static constexpr uint32_t SMALL = G + 73728;
  static constexpr uint32_t BETA = SMALL;                         // float [64]
  static constexpr uint32_t DVEC = SMALL + 256;                   // float [128]
  static constexpr uint32_t CST = SMALL + 768;                    // float [2][6][128] gate factors
  static constexpr uint32_t BAR = CST + 6144;                     // mbarrier: MMA completion
  static constexpr uint32_t TBAR = BAR + 8;                       // mbarrier: TMA loads landed
  static constexpr uint32_t SBAR = BAR + 16;                      // mbarrier: state product done
  static constexpr uint32_t TMEM_SLOT = BAR + 24;
  static constexpr uint32_t TOTAL = BAR + 64;
  static_assert(MT + 32 * 33 * 4 <= G + 65536, "solve scratch overflows");
  static_assert(64 * DVS * 2 <= 16384, "U must fit the Ktilde slot");
};

// Start loading the raw inputs of the chunk [t0, t0 + L): q, k, g into the
// staging area and v into its operand slot (one elected thread, TMA); beta
// into s_beta (64 threads, 4-byte async copies, zero past L).
template <int DVS>
__device__ __forceinline__ void prefetch_chunk(uint32_t sb, const TmaMaps &maps, const float *beta,
                                               int64_t t0, int L, int H, int h, int col0,
                                               int tid) {
  using Lay = Layout<DVS>;
  if (tid == 32) {   // not thread 0, which issues the tensor-core work
    const uint32_t bar = sb + Lay::TBAR;
    mbar_expect_tx(bar, 64 * (256 + 256 + 512) + 64 * DVS * 2);
    const int z = (int)t0;
    tma_load_3d(sb + Lay::STG_Q, &maps.q, 0, h, z, bar);
    tma_load_3d(sb + Lay::STG_K, &maps.k, 0, h, z, bar);
    tma_load_3d(sb + Lay::STG_G, &maps.g, 0, h, z, bar);
#pragma unroll
    for (int j = 0; j < DVS / 64; ++j)
      tma_load_3d(sb + Lay::KV_T + (2 + j) * 8192, &maps.v, col0 + 64 * j, h, z, bar);
  }
  if (tid >= 64 && tid < 64 + kC) {   // warps 2-3: thread 0 is left free for the MMAs
    const int r = tid - 64;
    const bool ok = r < L;
    cp_async4(sb + Lay::BETA + 4 * r, beta + (ok ? (size_t)(t0 + r) * H + h : 0), ok);
  }
  cp_async_commit();
}

template <int DVS>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ TmaMaps maps, const float *__restrict__ beta, const float *__restrict__ init,
                  const int32_t *__restrict__ cu, __nv_bfloat16 *__restrict__ out,
                  float *__restrict__ fin, int64_t interval, float *__restrict__ ck,
                  const int32_t *__restrict__ pos_cu, const int32_t *__restrict__ positions,
                  float *__restrict__ pos_states, int H, int32_t *dev_status, uint64_t wait_ns) {
  using Lay = Layout<DVS>;
  constexpr int NCOL = DVS / 2;           // state columns per thread
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t *sp = smem_raw + (sb - sraw);
  float *s_beta = reinterpret_cast<float *>(sp + Lay::BETA);
  float *s_dvec = reinterpret_cast<float *>(sp + Lay::DVEC);
  float *s_red = reinterpret_cast<float *>(sp + Lay::RED);
  float *s_cst = reinterpret_cast<float *>(sp + Lay::CST);
  float *s_M = reinterpret_cast<float *>(sp + Lay::MM);
  float *s_X = reinterpret_cast<float *>(sp + Lay::XM);
  float *s_Y = reinterpret_cast<float *>(sp + Lay::YS);
  float *s_Z = reinterpret_cast<float *>(sp + Lay::ZS);
  float *s_MT = reinterpret_cast<float *>(sp + Lay::MT);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sp + Lay::BAR);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hw = warp >> 2;      // TMEM lane quadrant, column half
  const int unit = blockIdx.x, seq = unit / H, h = unit % H;
  const int col0 = blockIdx.y * DVS;            // first value column of the slice
  const int crow = 32 * qd + lane;              // state row (key channel) owned

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(reinterpret_cast<uint64_t *>(sp + Lay::TBAR), 1);
    mbar_init(reinterpret_cast<uint64_t *>(sp + Lay::SBAR), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.q)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.g)) : "memory");
  }
  if (warp == 0) tc::tmem_alloc(sb + Lay::TMEM_SLOT, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + Lay::TMEM_SLOT);
  const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);   // this warp's lane base

  // The FP32 state slice lives in tensor memory, columns [128, 128 + DVS): lane c holds
  // state row c.  This thread owns row crow, columns [hw*NCOL, hw*NCOL + NCOL).
  const uint32_t s_tm = tl + 128 + hw * NCOL;
  const size_t soff = ((size_t)unit * kDK + crow) * kDV + col0 + hw * NCOL;
#pragma unroll
  for (int u = 0; u < NCOL / 32; ++u) {
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 v4 = init ? *reinterpret_cast<const float4 *>(init + soff + 32 * u + j)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      x[j] = v4.x; x[j + 1] = v4.y; x[j + 2] = v4.z; x[j + 3] = v4.w;
    }
    tc::tmem_st32(s_tm + 32 * u, x);
#pragma unroll
    for (int j = 0; j < 32; j += 8)
      tc::st_chunk(sb + Lay::S_T + tc::tile_offset(128, crow, (hw * NCOL + 32 * u + j) >> 3), x + j);
  }
  tc::tmem_wait_st();

  const int64_t t_begin = cu[seq], t_end = cu[seq + 1], T_seq = t_end - t_begin;
  int64_t ck_slot = 0;
  if (interval > 0)
    for (int j = 0; j < seq; ++j) ck_slot += (int64_t)(cu[j + 1] - cu[j]) / interval;
  // Explicit state positions of this sequence (token counts), if any.
  int pi = positions ? pos_cu[seq] : 0;
  const int pe = positions ? pos_cu[seq + 1] : 0;
  // Store the FP32 state slice of this thread (read back from tensor memory) into
  // a [.., H, D_k, D_v] array.
  auto store_state = [&](float *base_ptr, int64_t slot) {
    float *dst = base_ptr + ((size_t)slot * H + h) * kDK * kDV + (size_t)crow * kDV + col0 + hw * NCOL;
#pragma unroll
    for (int u = 0; u < NCOL / 32; ++u) {
      float x[32];
      tc::tmem_ld32(s_tm + 32 * u, x);
      tc::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4 *>(dst + 32 * u + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
    }
  };
  // Length of the chunk that starts after `done` tokens: at most 64, and it ends
  // at the next checkpoint boundary or explicit position (chunking does not
  // change the result, so every stored state is the state at a chunk end).
  // since_ck = done % interval is tracked incrementally (no 64-bit division in the loop).
  auto chunk_len = [&](int64_t done, int64_t since_ck, int p) -> int {
    int64_t m = T_seq - done < kC ? T_seq - done : kC;
    if (interval > 0) {
      const int64_t to_ck = interval - since_ck;
      m = to_ck < m ? to_ck : m;
    }
    if (p < pe) {
      const int64_t to_pos = (int64_t)positions[p] - done;
      m = to_pos < m ? to_pos : m;
    }
    return (int)m;
  };
  while (pi < pe && positions[pi] <= 0) store_state(pos_states, pi++);   // initial state

  uint32_t phase = 0, tphase = 0, sphase = 0;
  bool aborted = false;
  uint64_t *tbar = reinterpret_cast<uint64_t *>(sp + Lay::TBAR);
  uint64_t *sbar = reinterpret_cast<uint64_t *>(sp + Lay::SBAR);
  int64_t done = 0, since_ck = 0;
  int L = T_seq > 0 ? chunk_len(0, 0, pi) : 0;
  if (T_seq > 0) prefetch_chunk<DVS>(sb, maps, beta, t_begin, L, H, h, col0, tid);

  while (done < T_seq) {
    const int64_t t0 = t_begin + done;
    cp_async_wait_all();
    if (__syncthreads_or(!wait_timed(tbar, tphase, wait_ns))) { aborted = true; break; }
    tphase ^= 1;

    // ---------------- gate prep: cumulative decay and scaled operands ----------------
    // Warp w owns rows 8w..8w+7 (half hf = w / 4), lane l owns channels 4l..4l+3
    // (two pairs, on the paired FP32 instructions, each lane of which rounds like
    // the scalar one): per row one 8-byte piece of each 16-byte tile chunk; the
    // gate factors of the lane's channels stay in registers for all its rows.
    {
      const int hf = warp >> 2, cq = lane >> 1, sub = (lane & 1) * 8;
      float2 gm[8][2];
      uint2 kv[8], qv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * warp + i;
        const bool in = r < L;
        const float4 a = in ? *reinterpret_cast<const float4 *>(sp + Lay::STG_G + r * 512 + lane * 16)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        gm[i][0] = make_float2(a.x, a.y);
        gm[i][1] = make_float2(a.z, a.w);
        const uint2 z2 = make_uint2(0, 0);
        kv[i] = in ? *reinterpret_cast<const uint2 *>(sp + Lay::STG_K + r * 256 + lane * 8) : z2;
        qv[i] = in ? *reinterpret_cast<const uint2 *>(sp + Lay::STG_Q + r * 256 + lane * 8) : z2;
      }
#pragma unroll
      for (int i = 1; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) gm[i][j] = __fadd2_rn(gm[i][j], gm[i - 1][j]);
      *reinterpret_cast<float4 *>(s_red + warp * 128 + 4 * lane) =
          make_float4(gm[7][0].x, gm[7][0].y, gm[7][1].x, gm[7][1].y);
      __syncthreads();
      // One lane per channel: exclusive scan of the 8 row-group totals, the cumulative
      // decay at rows 15, 31, 47, 63 and the channel's gate factors for both halves.
      if (tid < 128) {
        const int ch = tid;
        float t[8], run = 0.f, incl[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = s_red[i * 128 + ch];
#pragma unroll
        for (int i = 0; i < 8; ++i) { run += t[i]; incl[i] = run; }
#pragma unroll
        for (int i = 0; i < 8; ++i) s_red[i * 128 + ch] = incl[i] - t[i];
        const float G15 = incl[1], G31 = incl[3], G47 = incl[5], G63 = incl[7];
        // Row r of half hf is scaled against ref = Gam_15 (hf 0) or Gam_47 (hf 1):
        // x = exp(Gam_r - ref), y = 1/x, both within [e^-80, e^80].  Products are
        // grouped so that an intermediate can only underflow when the exact value
        // is itself below e^-87 (or, for the B^(1) rows of the first half and
        // Ktilde of the second, below e^-12 times a unit-norm product).
        // Slots: -ref, fk, fk2, fh, fh2, cb; fk = 1 in the first half and fh2 = 1 in
        // the second, so (x fk) fk2 and (y fh) fh2 serve both halves exactly.
        float f[12];
        f[0] = -G15; f[1] = 1.f; f[2] = __expf(G15);
        f[3] = __expf(G31 - G15); f[4] = __expf(G63 - G31); f[5] = __expf(G47 - G15);
        f[6] = -G47; f[7] = __expf(G47 - G31); f[8] = __expf(G31);
        f[9] = __expf(G63 - G47); f[10] = 1.f; f[11] = 0.f;
#pragma unroll
        for (int j = 0; j < 12; ++j) s_cst[j * 128 + ch] = f[j];
        s_dvec[ch] = __expf(G63);
      }
      __syncthreads();
      float2 nref[2], fk[2], fk2[2], fh[2], fh2[2], cb[2];
      {
        auto ld4 = [&](int j, float2 *d) {
          const float4 v = *reinterpret_cast<const float4 *>(s_cst + (hf * 6 + j) * 128 + 4 * lane);
          d[0] = make_float2(v.x, v.y);
          d[1] = make_float2(v.z, v.w);
        };
        const float4 bv = *reinterpret_cast<const float4 *>(s_red + warp * 128 + 4 * lane);
        const float2 base[2] = {make_float2(bv.x, bv.y), make_float2(bv.z, bv.w)};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 2; ++j) gm[i][j] = __fadd2_rn(gm[i][j], base[j]);
        ld4(0, nref); ld4(1, fk); ld4(2, fk2); ld4(3, fh); ld4(4, fh2); ld4(5, cb);
      }
      auto st4 = [&](uint32_t off, const float2 *x) {
        *reinterpret_cast<uint2 *>(sp + off) = make_uint2(tc::pack_bf16(x[0].x, x[0].y), tc::pack_bf16(x[1].x, x[1].y));
      };
      auto un4 = [&](const uint2 &u, float2 *x) {
        x[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        x[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
      };
      auto rcp = [](float v) {   // hardware reciprocal approximation; v is normal here
        float r;
        asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
        return r;
      };
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * warp + i;
        float2 kk[2], qq[2], x[2], y[2], t[2];
        un4(kv[i], kk);
        un4(qv[i], qq);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float2 d = __fadd2_rn(gm[i][j], nref[j]);
          x[j] = make_float2(__expf(d.x), __expf(d.y));
          y[j] = make_float2(rcp(x[j].x), rcp(x[j].y));
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(kk[j], x[j]);
        st4(Lay::GA + tc::tile_offset(128, r, cq) + sub, t);
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(qq[j], x[j]);
        st4(Lay::GA + tc::tile_offset(128, 64 + r, cq) + sub, t);
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(kk[j], y[j]);
        st4(Lay::GB + tc::tile_offset(96, hf ? 32 + r : r, cq) + sub, t);
        if (!hf) {
#pragma unroll
          for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(kk[j], __fmul2_rn(y[j], cb[j]));
          st4(Lay::GB + tc::tile_offset(96, 32 + r, cq) + sub, t);
        }
        // Ktilde, Qtilde: exp(Gam_r) = (x fk) fk2.
#pragma unroll
        for (int j = 0; j < 2; ++j) x[j] = __fmul2_rn(__fmul2_rn(x[j], fk[j]), fk2[j]);
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(kk[j], x[j]);
        st4(Lay::WQ_T + tc::tile_offset(128, r, cq) + sub, t);
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(qq[j], x[j]);
        st4(Lay::WQ_T + tc::tile_offset(128, 64 + r, cq) + sub, t);
        // Khat: exp(Gam_63 - Gam_r) = (y fh) fh2.
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(kk[j], __fmul2_rn(__fmul2_rn(y[j], fh[j]), fh2[j]));
        st4(Lay::KH_T + tc::tile_offset(64, r, cq) + sub, t);
      }
      tc::fence_smem_to_async();
      __syncthreads();
    }

    // ---------------- gated Gram products: one [128 x 96 x 128] MMA ----------------
    // A = [k_r x_r ; q_r x_r] (rows 0..63 k, 64..127 q), B = [k_i exp(Gam_15 - Gam_i), i < 32 |
    // k_i exp(Gam_47 - Gam_i), i < 64].  Rows of the first half use columns 0..31, rows of
    // the second half columns 32..95; the other products are never read.
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 96, 0, 0);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem, tc::desc_kmajor(sb + Lay::GA, 128, s2), tc::desc_kmajor(sb + Lay::GB, 96, s2),
                     id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
      // The state product needs only prep's output and S0: [Ktilde; Qtilde] S0 -> acc1.
      // It completes on its own barrier, while the Gram rows are read and inverted.
      constexpr uint32_t id1 = tc::idesc_bf16(128, DVS, 0, 1);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem + 256, tc::desc_kmajor(sb + Lay::WQ_T, 128, s2),
                     tc::desc_mnmajor(sb + Lay::S_T, 128, s2), id1, s2 > 0);
      tc::mma_commit(sb + Lay::SBAR);
    }
    if (__syncthreads_or(!wait_timed(bar, phase, wait_ns))) { aborted = true; break; }
    phase ^= 1;
    tc::fence_after_sync();

    // Read the Gram rows: lane m = row m.  k-part rows become rows of the FP32 matrix M
    // (scaled by beta_r, strictly lower); q-part rows become rows of P, written straight
    // into rows 64..127 of the bf16 [T; P] operand.
    {
      const int m = 32 * qd + lane, part = m >> 6, r = m & 63, second = r >> 5;
      // first-half rows: hw 0 reads columns 0..31, hw 1 writes the zero half;
      // second-half rows: hw 0 reads i = 0..31 (columns 32..63), hw 1 i = 32..63.
      const int i0 = second ? 32 * hw : (hw ? 32 : 0);
      float a[32];
      if (second || hw == 0) {
        tc::tmem_ld32(tl + (second ? 32 + 32 * hw : 0), a);
        tc::tmem_wait_ld();
      }
      const bool zero = !second && hw;
      if (part == 0) {
        const float br = s_beta[r];
        float *dst = s_M + r * kLd + i0;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[j] = (!zero && i0 + j < r) ? br * a[j] : 0.f;
        if (second && i0 == 0)   // the block M_(1,0), also transposed for the solve
#pragma unroll
          for (int j = 0; j < 32; ++j) s_MT[j * 33 + (r - 32)] = br * a[j];
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) a[j] = (!zero && i0 + j <= r) ? a[j] : 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          tc::st_chunk(sb + Lay::TP_T + tc::tile_offset(128, 64 + r, (i0 >> 3) + cc), a + 8 * cc);
      }
    }
    tc::fence_before_sync();
    __syncthreads();

    // ---------------- UT transform: X = (I + M)^-1, blockwise on 16x16 blocks ----------------
    // Diagonal blocks: warp b inverts block b by a column sweep; lane = (column c,
    // half hf) holds rows 8hf..8hf+7 of column c; row s is broadcast by shuffle.
    if (qd >= 2) {   // warps 2, 3, 6, 7 invert the diagonal blocks 0, 1, 2, 3
      const int blk = (qd - 2) + 2 * hw;
      const int o = 16 * blk, c = lane & 15, hf = lane >> 4;
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = (8 * hf + i == c) ? 1.f : 0.f;
      const float *mrow = s_M + (o + 8 * hf) * kLd + o;
#pragma unroll
      for (int sidx = 0; sidx < 15; ++sidx) {
        float m[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = mrow[i * kLd + sidx];   // 0 on and above the diagonal
        const float xs = __shfl_sync(0xffffffffu, x[sidx & 7], c + 16 * (sidx >> 3));
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = fmaf(-m[i], xs, x[i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) s_X[(o + 8 * hf + i) * kLd + o + c] = x[i];
      if ((blk & 1) == 0)   // block above the diagonal inside the 32-row half
#pragma unroll
        for (int i = 0; i < 8; ++i) s_X[(o + 8 * hf + i) * kLd + o + 16 + c] = 0.f;
    }
    // Meanwhile warps 0, 1, 4, 5 (TMEM lanes 0..63) form X = V - Ktilde S0 for tokens
    // 0..63 from the state product and write it as the bf16 operand of U = T X.
    bool s_late = false;
    if (qd < 2) {
      s_late = !wait_timed(sbar, sphase, wait_ns);
      tc::fence_after_sync();
      const int r = 32 * qd + lane;
#pragma unroll
      for (int col = hw * NCOL; col < hw * NCOL + NCOL; col += 32) {
        float a[32];
        tc::tmem_ld32(tl + 256 + col, a);
        tc::tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint4 vv = *reinterpret_cast<const uint4 *>(
              sp + Lay::KV_T + tc::tile_offset(64, r, 16 + (col >> 3) + cc));
          float xv[8];
          unpack8(vv, xv);
#pragma unroll
          for (int e = 0; e < 8; ++e) xv[e] -= a[8 * cc + e];
          tc::st_chunk(sb + Lay::U_T + tc::tile_offset(64, r, (col >> 3) + cc), xv);
        }
      }
      tc::fence_smem_to_async();
      tc::fence_before_sync();
    }
    if (__syncthreads_or(s_late)) { aborted = true; break; }
    sphase ^= 1;
    // Level 1: the 32x32 inverse of each half, X_(2h+1,2h) = -X_(2h+1,2h+1) M_(2h+1,2h) X_(2h,2h).
    {
      const int hh = tid >> 7, rr = (tid >> 3) & 15, c0 = (tid & 7) * 2;
      const int ro = 32 * hh + 16, co = 32 * hh;
      float y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int s2 = 0; s2 < 16; ++s2) {
        const float m = s_M[(ro + rr) * kLd + co + s2];
        const float2 xv = *reinterpret_cast<const float2 *>(s_X + (co + s2) * kLd + co + c0);
        y0 = fmaf(m, xv.x, y0);
        y1 = fmaf(m, xv.y, y1);
      }
      s_Y[(hh * 16 + rr) * 17 + c0] = y0;
      s_Y[(hh * 16 + rr) * 17 + c0 + 1] = y1;
      __syncthreads();
      float x0 = 0.f, x1 = 0.f;
#pragma unroll
      for (int s2 = 0; s2 < 16; ++s2) {
        const float a = s_X[(ro + rr) * kLd + ro + s2];
        x0 = fmaf(a, s_Y[(hh * 16 + s2) * 17 + c0], x0);
        x1 = fmaf(a, s_Y[(hh * 16 + s2) * 17 + c0 + 1], x1);
      }
      *reinterpret_cast<float2 *>(s_X + (ro + rr) * kLd + co + c0) = make_float2(-x0, -x1);
      __syncthreads();
    }
    // Level 2: X_(1,0) = -H1 M_(1,0) H0 on the 32x32 halves.  H0 and H1 are lower
    // triangular, so each warp's trip count skips the zero half of the product.
    {
      // Z = M_(1,0) H0: warp w computes columns 4w..4w+3, lane = row; H0[s][c] = 0 for s < c.
      const int rr = lane, cq = 4 * warp;
      float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s2 = cq; s2 < 32; ++s2) {
        const float m = s_MT[s2 * 33 + rr];
        const float4 xv = *reinterpret_cast<const float4 *>(s_X + s2 * kLd + cq);
        z.x = fmaf(m, xv.x, z.x); z.y = fmaf(m, xv.y, z.y);
        z.z = fmaf(m, xv.z, z.z); z.w = fmaf(m, xv.w, z.w);
      }
      *reinterpret_cast<float4 *>(s_Z + rr * 36 + cq) = z;
      __syncthreads();
      // X_(1,0) = -H1 Z: warp w computes rows 4w..4w+3; H1[r][s] = 0 for s > r.
      const int r2 = 4 * warp + (lane >> 3), c2 = 4 * (lane & 7);
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s2 = 0; s2 < 4 * warp + 4; ++s2) {
        const float a = s_X[(32 + r2) * kLd + 32 + s2];
        const float4 zv = *reinterpret_cast<const float4 *>(s_Z + s2 * 36 + c2);
        w.x = fmaf(a, zv.x, w.x); w.y = fmaf(a, zv.y, w.y);
        w.z = fmaf(a, zv.z, w.z); w.w = fmaf(a, zv.w, w.w);
      }
      *reinterpret_cast<float4 *>(s_X + (32 + r2) * kLd + c2) = make_float4(-w.x, -w.y, -w.z, -w.w);
      __syncthreads();
    }
    // T rows of the [T; P] operand: T_ri = X_ri beta_i (i <= r).
    for (int e = tid; e < 64 * 8; e += kThreads) {
      const int row = e >> 3, ch = e & 7;
      float val[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = 8 * ch + u;
        val[u] = i <= row ? s_X[row * kLd + i] * s_beta[i] : 0.f;
      }
      tc::st_chunk(sb + Lay::TP_T + tc::tile_offset(128, row, ch), val);
    }
    tc::fence_smem_to_async();
    __syncthreads();

    // Prefetch the next chunk: the staging area and the V slot are free now.
    const int64_t done_next = done + L;
    int p_next = pi;
    while (p_next < pe && positions[p_next] <= done_next) ++p_next;
    int64_t since_next = since_ck + L;
    if (since_next == interval) since_next = 0;
    const int L_next = done_next < T_seq ? chunk_len(done_next, since_next, p_next) : 0;
    if (done_next < T_seq)
      prefetch_chunk<DVS>(sb, maps, beta, t_begin + done_next, L_next, H, h, col0, tid);

    // ---------------- U = T X (rows 0..63 of [T; P] X) ----------------
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, DVS, 0, 1);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem, tc::desc_kmajor(sb + Lay::TP_T, 128, s2),
                     tc::desc_mnmajor(sb + Lay::U_T, 64, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (__syncthreads_or(!wait_timed(bar, phase, wait_ns))) { aborted = true; break; }
    phase ^= 1;
    tc::fence_after_sync();
    if (qd < 2) {   // U -> bf16 operand (replaces X, which the MMA has consumed)
      const int r = 32 * qd + lane;
      float a[32];
#pragma unroll
      for (int u = 0; u < NCOL / 32; ++u) {
        const int col = hw * NCOL + 32 * u;
        tc::tmem_ld32(tl + col, a);
        tc::tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          tc::st_chunk(sb + Lay::U_T + tc::tile_offset(64, r, (col >> 3) + cc), a + 8 * cc);
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();

    // ---------------- MMA2: O += P U, dS = Khat^T U ----------------
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t ida = tc::idesc_bf16(128, DVS, 0, 1);
      constexpr uint32_t idb = tc::idesc_bf16(128, DVS, 1, 1);
#pragma unroll
      for (int s = 0; s < 4; ++s)
        tc::mma_bf16(tmem + 256, tc::desc_kmajor(sb + Lay::TP_T, 128, s),
                     tc::desc_mnmajor(sb + Lay::U_T, 64, s), ida, 1);
#pragma unroll
      for (int s = 0; s < 4; ++s)
        tc::mma_bf16(tmem + 256 + DVS, tc::desc_mnmajor(sb + Lay::KH_T, 64, s),
                     tc::desc_mnmajor(sb + Lay::U_T, 64, s), idb, s > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (__syncthreads_or(!wait_timed(bar, phase, wait_ns))) { aborted = true; break; }
    phase ^= 1;
    tc::fence_after_sync();
    {
      float a[32];
      if (qd >= 2) {   // rows 64..127 hold O for tokens 0..63
        const int r = 32 * (qd - 2) + lane;
#pragma unroll
        for (int u = 0; u < NCOL / 32; ++u) {
          const int col = hw * NCOL + 32 * u;
          tc::tmem_ld32(tl + 256 + col, a);
          tc::tmem_wait_ld();
          if (r < L) {
            uint4 *dst = reinterpret_cast<uint4 *>(out + ((size_t)(t0 + r) * H + h) * kDV + col0 + col);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              dst[cc] = make_uint4(tc::pack_bf16(a[8 * cc], a[8 * cc + 1]),
                                   tc::pack_bf16(a[8 * cc + 2], a[8 * cc + 3]),
                                   tc::pack_bf16(a[8 * cc + 4], a[8 * cc + 5]),
                                   tc::pack_bf16(a[8 * cc + 6], a[8 * cc + 7]));
          }
        }
      }
      const float d = s_dvec[crow];
#pragma unroll
      for (int u = 0; u < NCOL / 32; ++u) {
        float sv[32];
        tc::tmem_ld32(tl + 256 + DVS + hw * NCOL + 32 * u, a);   // state increment
        tc::tmem_ld32(s_tm + 32 * u, sv);                          // state
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[i] = fmaf(d, sv[i], a[i]);
        tc::tmem_st32(s_tm + 32 * u, sv);
#pragma unroll
        for (int j = 0; j < 32; j += 8)
          tc::st_chunk(sb + Lay::S_T + tc::tile_offset(128, crow, (hw * NCOL + 32 * u + j) >> 3), sv + j);
      }
      tc::tmem_wait_st();
      done += L;
      since_ck += L;
      if (interval > 0 && since_ck == interval) {
        store_state(ck, ck_slot++);
        since_ck = 0;
      }
      while (pi < pe && positions[pi] <= done) store_state(pos_states, pi++);
      L = L_next;
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
  }

  cp_async_wait_all();
  if (aborted) {
    report(dev_status, KDA_ERR_TIMEOUT);
    // Give the tensor core and the copy engine a last bounded chance to finish
    // what they were given before the CTA releases its memory.
    wait_timed(bar, phase, wait_ns);
    wait_timed(sbar, sphase, wait_ns);
    wait_timed(tbar, tphase, wait_ns);
  } else {
    while (pi < pe) store_state(pos_states, pi++);   // positions past the end: final state
    if (fin) store_state(fin, seq);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int DVS>
cudaError_t launch_tc_t(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *init, const int32_t *cu, void *out,
                        float *fin, int64_t interval, float *ck, const int32_t *pos_cu,
                        const int32_t *positions, float *pos_states, int N, int H, int64_t T,
                        int32_t *dev_status, cudaStream_t stream) {
  TmaMaps maps;
  if (!make_input_maps(&maps, q, k, v, g, H, T)) return cudaErrorInvalidValue;
  const size_t smem = Layout<DVS>::TOTAL + 1024;
  auto kern = prefill_tc_kernel<DVS>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)((int64_t)N * H), (unsigned)(kDV / DVS));
  kern<<<grid, kThreads, smem, stream>>>(maps, beta, init, cu, (__nv_bfloat16 *)out, fin, interval,
                                         ck, pos_cu, positions, pos_states, H, dev_status,
                                         2000000000ull);
  return cudaGetLastError();
}

}  // namespace

bool prefill_tc_supported(int dtype, int dk, int dv, int chunk) {
  return dtype == KDA_DTYPE_BF16 && dk == kDK && dv == kDV && chunk == kC;
}

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *init, const int32_t *cu, void *out,
                              float *fin, int64_t interval, float *ck, const int32_t *pos_cu,
                              const int32_t *positions, float *pos_states, int N, int H,
                              int64_t total_tokens, int32_t *dev_status, cudaStream_t stream) {
  // Few (sequence, head) units: split the value columns in two to fill the SMs.
  if ((int64_t)N * H * 2 <= 148)
    return launch_tc_t<64>(q, k, v, g, beta, init, cu, out, fin, interval, ck, pos_cu, positions,
                           pos_states, N, H, total_tokens, dev_status, stream);
  return launch_tc_t<128>(q, k, v, g, beta, init, cu, out, fin, interval, ck, pos_cu, positions,
                          pos_states, N, H, total_tokens, dev_status, stream);
}

}  // namespace kda
