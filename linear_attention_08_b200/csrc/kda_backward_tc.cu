// Backward pass of KDA on the 5th-generation tensor cores (tcgen05, sm_100a),
// for BF16 q/k/v with D_k = D_v = 128: the chunked form of the gradients.
//
// The pages name training work without detail ("MoonshotAI/Kimi-K3 딥다이브",
// section 4-1); the gradients below follow from the chunked forward
// ("LLM - Semianalysis, Kimi K3 아키텍처", Methods 1: intra-chunk matrix
// products plus a recurrence between chunks) by reverse-mode differentiation.
// For one chunk (64 tokens, padded with identity tokens) starting from S0,
// with Gam_r the inclusive cumulative log-decay inside the chunk,
// Ktilde = k e^Gam, Qtilde = q e^Gam, Khat = k e^(Gam_63 - Gam), d = e^Gam_63,
// the gated Gram G_ij = sum_c k_ic k_jc e^(Gam_ic - Gam_jc) (j < i),
// P_ri = sum_c q_rc k_ic e^(Gam_rc - Gam_ic) (i <= r), A = I + diag(beta) G,
// Ai = A^-1, T = Ai diag(beta):
//
//   R = V - Ktilde S0,  U = T R,  O = Qtilde S0 + P U,
//   S_L = Diag(d) S0 + Khat^T U.
//
// Given dO and dS_L (the gradient of the state at the chunk's end):
//
//   dU  = P^T dO + Khat dS_L          dR = T^T dU = dV        dT = dU R^T
//   dP  = dO U^T                      dQtilde = dO S0^T       dKtilde = -dR S0^T
//   dKhat = U dS_L^T                  dd_c = sum_j dS_L[c,j] S0[c,j]
//   dS0 = Diag(d) dS_L + Qtilde^T dO - Ktilde^T dR
//       = Diag(d) dS_L + Qtilde^T dO - W^T dU        (W = T Ktilde)
//   Y1 = Ai^T dT: dbeta_j += Y1_jj;   dA = -Y1 T^T, dM = strict lower part,
//   dbeta_i += sum_j dM_ij G_ij,  dG_ij = beta_i dM_ij,
//
// and the gated products G, P, Qtilde, Ktilde, Khat, d pass their gradients to
// q, k and Gam; dg is the reverse cumulative sum of dGam inside the chunk.
//
// The forward is recomputed first (the two-pass prefill, keeping its
// intra-chunk packets, each chunk's T and Ai as BF16 tiles, and the state at
// every chunk end as a BF16 tile); small launches then build the item prefix
// and the BF16 tiles of dO and of the initial states.  Then:
//  1. bwd_chain_kernel: one CTA per (sequence, head) walks the chunks
//     backwards carrying dS in tensor memory: per chunk dU = [Khat | P^T]
//     [dS; dO] and dS <- d dS + [W^T | Qtilde^T] [-dU; dO], two tcgen05 MMAs.
//     It stores dS_L and -dU per chunk as BF16 tiles.
//  2. bwd_item_kernel<0>, the state part (per (chunk, head), persistent):
//     recomputes Gam and Ktilde, takes T from the forward, then R, U,
//     dR (= dv), dT, dP, dQtilde, dKtilde, dKhat and dd on the tensor cores;
//     writes dv and the parts of dq, dk and dg those terms give, and dT, dP.
//  3. bwd_item_kernel<1>, the Gram part: recomputes the gates and G, takes T
//     and Ai from the forward, then Y1, dA, dG and the gated products of dG
//     and dP on the tensor cores; adds the rest of dq, dk, dg (global
//     reductions) and writes dbeta.
#include <cuda.h>

#include "kda_common.cuh"
#include "kda_tc_util.cuh"
#include "kda_tma.cuh"

namespace kda {

cudaError_t launch_prefill_split_ex(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const float *init, const int32_t *cu,
                                    void *out, float *fin, int64_t interval, float *ck,
                                    uint8_t *ck_tiles, uint8_t *tt_out, int N, int H, int64_t T,
                                    void *workspace, size_t ws_bytes, int32_t *dev_status,
                                    cudaStream_t stream, int num_sms);
size_t split_packet_bytes();
bool prefill_split_supported(int N);

namespace {

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 256;

// The packet the forward intra-chunk pass writes per (chunk, head): operand
// tiles in the 128-byte-swizzled row-tile layout of kda_tc_util.cuh.
struct Pk {
  static constexpr uint32_t WQ = 0;        // [128][128]: W rows 0..63, Qtilde rows 64..127
  static constexpr uint32_t KH = 32768;    // [64][128] Khat (tokens x key channels)
  static constexpr uint32_t P = 65536;     // [64][64] P, lower triangle with diagonal, then
                                           // float[128] exp(Gam_63) at 73728
  static constexpr uint32_t BYTES = 74240;
};

// Where packet p sits: written by the dO tile conversion, which locates every
// packet anyway, and read by the per-chunk kernels with one independent load
// instead of a search and divisions on each item's path.
struct ItemRec {
  int64_t t0, j;   // first token, chunk index in the sequence
  int32_t n, h, L, pad;
};

// Chunks of sequence n.
__device__ __forceinline__ int64_t seq_chunks(const int32_t *cu, int n) {
  return ((int64_t)cu[n + 1] - cu[n] + kC - 1) / kC;
}

// ---------------------------------------------------------------------------
// 1. The backward chain
// ---------------------------------------------------------------------------
struct BChainLayout {
  static constexpr uint32_t S_T = 0;         // [128 ch][128 v] bf16 dS, MN-major B (stored as dS_L)
  static constexpr uint32_t NDU = 32768;     // [64 tok][128 v] bf16 -dU, MN-major B (stored)
  static constexpr uint32_t STAGE0 = 49152;  // stages: a chunk's packet and its dO tile
  // Inside a stage.  Khat and P come first: the M = 128 MMAs that read them as
  // 64-row operands also read the 8 KB after each (rows 64..127 of the
  // product, never used), which must stay inside the stage.
  static constexpr uint32_t SKH = 0;         // [64][128] Khat
  static constexpr uint32_t SP = 16384;      // [64][64] P
  static constexpr uint32_t SD = 24576;      // float[128] d
  static constexpr uint32_t SWQ = 25600;     // [128][128] [W; Qtilde]
  static constexpr uint32_t SDO = SWQ + 32768;   // [64 tok][128 v] bf16 dO, MN-major B
  static constexpr uint32_t STAGE = SDO + 16384;
  static constexpr int NST = 2;
  static constexpr uint32_t FULL = STAGE0 + NST * STAGE;   // [NST] stage landed
  static constexpr uint32_t BAR1 = FULL + 8 * NST;         // dU product done
  static constexpr uint32_t BAR2 = BAR1 + 8;               // dS product done
  static constexpr uint32_t SCAL = BAR2 + 8;               // int64 first packet of the unit
  static constexpr uint32_t TMEM_SLOT = SCAL + 8;
  static constexpr uint32_t TOTAL = TMEM_SLOT + 8;
  static constexpr uint32_t TX = 16384 + 8704 + 32768 + 16384;   // bytes landing per stage
  static constexpr uint32_t ACC1 = 0, ACC2 = 128, SCOL = 256;   // TMEM columns
  static_assert(SKH + 16384 + 8192 <= STAGE && SP + 8192 + 8192 <= STAGE, "junk rows leave the stage");
  static_assert(STAGE % 1024 == 0 && SWQ % 1024 == 0 && SDO % 1024 == 0, "tile alignment");
  static_assert(TOTAL + 1024 <= 232448, "shared memory");
};

// The chunk's dO as the BF16 operand tile [64 tokens][128 value columns]
// (rows past the sequence's end zero), for every packet: two packets per CTA.
__global__ void __launch_bounds__(kThreads)
bwd_dout_tiles_kernel(const float *__restrict__ dout, const int32_t *__restrict__ cu,
                      const int64_t *__restrict__ pref, int N, int H, uint8_t *__restrict__ tiles,
                      ItemRec *__restrict__ items) {
  // Two items per CTA: both items' rows are loaded before any store.  Warp w
  // takes rows w, w + 8, .., lane l columns 4l .. 4l + 3: every load is one
  // whole 512-byte row of dO.
  const int64_t total = pref[N] * H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, c = 4 * lane;
  float4 x[2][8];
  int64_t pp[2];
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int64_t p = 2 * (int64_t)blockIdx.x + it;
    pp[it] = p;
    int L = 0;
    const float *src = dout;
    size_t stride = 0;
    if (p < total) {
      int lo = 0, hi = N - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pref[mid] * H <= p) lo = mid; else hi = mid - 1;
      }
      const int n = lo;
      const int64_t nch = pref[n + 1] - pref[n];
      const int64_t rem = p - pref[n] * H;
      const int h = (int)(rem / nch);
      const int64_t j = rem - (int64_t)h * nch;
      const int64_t t0 = (int64_t)cu[n] + kC * j;
      const int64_t T_n = (int64_t)cu[n + 1] - cu[n];
      L = (int)(T_n - kC * j < kC ? T_n - kC * j : kC);
      if (tid == 0) {
        ItemRec rec;
        rec.t0 = t0; rec.j = j; rec.n = n; rec.h = h; rec.L = L; rec.pad = 0;
        items[p] = rec;
      }
      src = dout + ((size_t)t0 * H + h) * kD + c;
      stride = (size_t)H * kD;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = warp + 8 * i;
      x[it][i] = r < L ? *reinterpret_cast<const float4 *>(src + (size_t)r * stride)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    if (pp[it] >= total) continue;
    uint8_t *dst = tiles + (size_t)pp[it] * 16384 + 2 * (c & 7);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint2 *>(dst + tc::tile_offset(64, warp + 8 * i, c >> 3)) =
          make_uint2(tc::pack_bf16(x[it][i].x, x[it][i].y), tc::pack_bf16(x[it][i].z, x[it][i].w));
  }
}

__global__ void __launch_bounds__(kThreads, 1)
bwd_chain_kernel(const uint8_t *__restrict__ pk, const uint8_t *__restrict__ dotiles,
                 const int32_t *__restrict__ cu, const float *__restrict__ dfin,
                 float *__restrict__ dinit, uint8_t *__restrict__ dsl, uint8_t *__restrict__ ndu,
                 int N, int H, int32_t *dev_status, uint64_t wait_ns) {
  using Lay = BChainLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t *sp = smem_raw + (sb - sraw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hw = warp >> 2;
  const int unit = blockIdx.x, n = unit / H, h = unit % H;
  const int crow = 32 * qd + lane;   // TMEM lane of this thread: a key channel
  const int64_t nch = seq_chunks(cu, n);

  if (warp == 0) {   // first packet of sequence n (packets: sequence, head, chunk)
    int64_t before = 0;
    for (int m = lane; m < n; m += 32) before += seq_chunks(cu, m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
    if (lane == 0) *reinterpret_cast<int64_t *>(sp + Lay::SCAL) = before;
  }
  uint64_t *full = reinterpret_cast<uint64_t *>(sp + Lay::FULL);
  uint64_t *bar1 = reinterpret_cast<uint64_t *>(sp + Lay::BAR1);
  uint64_t *bar2 = reinterpret_cast<uint64_t *>(sp + Lay::BAR2);
  if (tid == 0) {
    for (int s = 0; s < Lay::NST; ++s) mbar_init(full + s, 1);
    mbar_init(bar1, 1);
    mbar_init(bar2, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tc::tmem_alloc(sb + Lay::TMEM_SLOT, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + Lay::TMEM_SLOT);
  const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
  const int64_t p0 = *reinterpret_cast<const int64_t *>(sp + Lay::SCAL) * H + (int64_t)h * nch;

  auto issue_stage = [&](int64_t c, int s) {
    const uint8_t *src = pk + (size_t)(p0 + c) * Pk::BYTES;
    const uint32_t st = sb + Lay::STAGE0 + s * Lay::STAGE;
    const uint32_t fb = sb + Lay::FULL + 8 * s;
    mbar_expect_tx(fb, Lay::TX);
    bulk_load(st + Lay::SKH, src + Pk::KH, 16384, fb);
    bulk_load(st + Lay::SP, src + Pk::P, 8704, fb);      // P and d
    bulk_load(st + Lay::SWQ, src + Pk::WQ, 32768, fb);
    bulk_load(st + Lay::SDO, dotiles + (size_t)(p0 + c) * 16384, 16384, fb);
  };
  if (tid == 32)
    for (int s = 0; s < Lay::NST && s < nch; ++s) issue_stage(nch - 1 - s, s);

  // dS = dS_final, FP32 in tensor memory (lane = key channel), BF16 copy in S_T.
  const uint32_t s_tm = tl + Lay::SCOL + hw * 64;
  {
    const float *src = dfin ? dfin + ((size_t)unit * kD + crow) * kD + hw * 64 : nullptr;
    float *dst0 = (nch == 0 && dinit) ? dinit + ((size_t)unit * kD + crow) * kD + hw * 64 : nullptr;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float x[32];
#pragma unroll
      for (int jj = 0; jj < 32; jj += 4) {
        const float4 v4 = src ? *reinterpret_cast<const float4 *>(src + 32 * u + jj)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        x[jj] = v4.x; x[jj + 1] = v4.y; x[jj + 2] = v4.z; x[jj + 3] = v4.w;
        if (dst0) *reinterpret_cast<float4 *>(dst0 + 32 * u + jj) = v4;
      }
      tc::tmem_st32(s_tm + 32 * u, x);
#pragma unroll
      for (int jj = 0; jj < 32; jj += 8)
        tc::st_chunk(sb + Lay::S_T + tc::tile_offset(128, crow, (hw * 64 + 32 * u + jj) >> 3), x + jj);
    }
    tc::tmem_wait_st();
  }
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();
  if (tid == 0 && nch > 0) {   // dS_L of the last chunk
    bulk_store(dsl + (size_t)(p0 + nch - 1) * 32768, sb + Lay::S_T, 32768);
    bulk_commit();
  }

  uint32_t fphase = 0, ph1 = 0, ph2 = 0;
  bool aborted = false;
  for (int64_t i = 0; i < nch; ++i) {
    const int64_t c = nch - 1 - i;
    const int s = (int)(i % Lay::NST);
    const uint32_t st = sb + Lay::STAGE0 + s * Lay::STAGE;
    if (__syncthreads_or(!wait_timed(full + s, (fphase >> s) & 1u, wait_ns))) { aborted = true; break; }
    fphase ^= 1u << s;
    // acc1 = Khat dS + P^T dO  (rows 0..63: dU)
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t idk = tc::idesc_bf16(128, 128, 0, 1);
      constexpr uint32_t idm = tc::idesc_bf16(128, 128, 1, 1);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem + Lay::ACC1, tc::desc_kmajor(st + Lay::SKH, 64, s2),
                     tc::desc_mnmajor(sb + Lay::S_T, 128, s2), idk, s2 > 0);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + Lay::ACC1, tc::desc_mnmajor(st + Lay::SP, 64, s2),
                     tc::desc_mnmajor(st + Lay::SDO, 64, s2), idm, 1);
      tc::mma_commit(sb + Lay::BAR1);
      bulk_wait_read();   // the previous -dU and dS_L stores have left NDU and S_T
    }
    if (__syncthreads_or(!wait_timed(bar1, ph1, wait_ns))) { aborted = true; break; }
    ph1 ^= 1;
    tc::fence_after_sync();
    if (qd < 2) {   // -dU -> NDU
      const int r = 32 * qd + lane;
      float a[64];
      tc::tmem_ld32(tl + Lay::ACC1 + hw * 64, *reinterpret_cast<float(*)[32]>(a));
      tc::tmem_ld32(tl + Lay::ACC1 + hw * 64 + 32, *reinterpret_cast<float(*)[32]>(a + 32));
      tc::tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 64; ++jj) a[jj] = -a[jj];
#pragma unroll
      for (int jj = 0; jj < 64; jj += 8)
        tc::st_chunk(sb + Lay::NDU + tc::tile_offset(64, r, (hw * 64 + jj) >> 3), a + jj);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    // -dU goes to the workspace; acc2 = W^T (-dU) + Qtilde^T dO
    if (tid == 0) {
      tc::fence_after_sync();
      bulk_store(ndu + (size_t)(p0 + c) * 16384, sb + Lay::NDU, 16384);
      bulk_commit();
      constexpr uint32_t id = tc::idesc_bf16(128, 128, 1, 1);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + Lay::ACC2, tc::desc_mnmajor(st + Lay::SWQ, 128, s2),
                     tc::desc_mnmajor(sb + Lay::NDU, 64, s2), id, s2 > 0);
#pragma unroll
      for (int s2 = 4; s2 < 8; ++s2)
        tc::mma_bf16(tmem + Lay::ACC2, tc::desc_mnmajor(st + Lay::SWQ, 128, s2),
                     tc::desc_mnmajor(st + Lay::SDO, 64, s2 - 4), id, 1);
      tc::mma_commit(sb + Lay::BAR2);
    }
    const float dch = reinterpret_cast<const float *>(sp + (st - sb) + Lay::SD)[crow];
    if (__syncthreads_or(!wait_timed(bar2, ph2, wait_ns))) { aborted = true; break; }
    ph2 ^= 1;
    tc::fence_after_sync();
    {   // dS <- d dS + acc2: the gradient of the state at the end of chunk c - 1
      float a[64], sv[64];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        tc::tmem_ld32(tl + Lay::ACC2 + hw * 64 + 32 * u, *reinterpret_cast<float(*)[32]>(a + 32 * u));
        tc::tmem_ld32(s_tm + 32 * u, *reinterpret_cast<float(*)[32]>(sv + 32 * u));
      }
      tc::tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 64; ++jj) sv[jj] = fmaf(dch, sv[jj], a[jj]);
#pragma unroll
      for (int u = 0; u < 2; ++u) tc::tmem_st32(s_tm + 32 * u, *reinterpret_cast<float(*)[32]>(sv + 32 * u));
#pragma unroll
      for (int jj = 0; jj < 64; jj += 8)
        tc::st_chunk(sb + Lay::S_T + tc::tile_offset(128, crow, (hw * 64 + jj) >> 3), sv + jj);
      if (c == 0 && dinit) {
        float *dst = dinit + ((size_t)unit * kD + crow) * kD + hw * 64;
#pragma unroll
        for (int jj = 0; jj < 64; jj += 4)
          *reinterpret_cast<float4 *>(dst + jj) = make_float4(sv[jj], sv[jj + 1], sv[jj + 2], sv[jj + 3]);
      }
      tc::tmem_wait_st();
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && c > 0) {   // dS_L of chunk c - 1, as the BF16 tile
      bulk_store(dsl + (size_t)(p0 + c - 1) * 32768, sb + Lay::S_T, 32768);
      bulk_commit();
    }
    if (tid == 32 && c - Lay::NST >= 0) issue_stage(c - Lay::NST, s);
  }
  if (tid == 0) bulk_wait_all();
  if (aborted) {
    report(dev_status, KDA_ERR_TIMEOUT);
    wait_timed(bar1, ph1, wait_ns);
    wait_timed(bar2, ph2, wait_ns);
    for (int s = 0; s < Lay::NST; ++s) wait_timed(full + s, (fphase >> s) & 1u, wait_ns);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace
}  // namespace kda

namespace kda {
namespace {

// ---------------------------------------------------------------------------
// 2, 3. Per (chunk, head): the state part (PART 0) and the Gram part (PART 1)
// ---------------------------------------------------------------------------
struct BItemLayout {
  static constexpr uint32_t GA = 0;          // [128][128] Gram A: k x rows 0..63, q x rows 64..127
  static constexpr uint32_t S0T = GA;        //   PART 0 (no Gram tiles): S0 [ch][v] bf16
  static constexpr uint32_t GB = 32768;      // [96][128] Gram B: k y (ref 1) | k y (ref 2), first half | k y, second half
  static constexpr uint32_t RU = 32768;      //   PART 0: [U; R] [tok][v] bf16 (128 rows)
  static constexpr uint32_t GST = 65536;     // float [64][128]: g, then Gam in place
  static constexpr uint32_t KT = 98304;      // [64][128] k, then Ktilde in place (PART 0)
  static constexpr uint32_t VT = 114688;     // [64][128] V (PART 0)
  static constexpr uint32_t BT2 = KT;        //   PART 0, after R: [-dU; dO] from the chain, then [-dR; dO]
  static constexpr uint32_t XA = KT;         //   PART 1: [dG; dP] placed against Gram B (K = 96)
  static constexpr uint32_t MM = 131072;     // prep scan partials, then dS_L (PART 0) or [dG^T | dP^T] (PART 1)
  static constexpr uint32_t XM = MM + 17408; // gate factors during the prep
  static constexpr uint32_t CST = XM;        //   gate factors during the prep: float [2][6][128]
  static constexpr uint32_t DST = MM;        //   PART 0: dS_L [ch][v] bf16
  static constexpr uint32_t YA = MM;         //   PART 1: [dG^T | dP^T] placed against Gram A
  static constexpr uint32_t YS = XM + 17408; // float [2][256]: the reverse scan's partial sums
  static constexpr uint32_t ZS = YS + 2176;  // (free)
  static constexpr uint32_t MT = ZS + 4608;  // (free)
  static constexpr uint32_t GG = MT + 4224;  // float [64][68] G (PART 1)
  static constexpr uint32_t TT = 194560;     // [64][64] T (row r, column i) bf16, from the forward
  static constexpr uint32_t RED = MM;        //   scan partials during the prep: float [8][128]
  static constexpr uint32_t AIT = TT + 8192; // [64][64] (I + M)^-1 bf16, from the forward (PART 1)
  static constexpr uint32_t Y1T = AIT + 8192;// [64][64] Y1 = Ai^T dT bf16 (PART 1)
  static constexpr uint32_t DTT = Y1T + 8192;// [64][64] dT bf16 (PART 1)
  static constexpr uint32_t BETA = DTT + 8192;            // float [64]
  static constexpr uint32_t DD = BETA + 256;              // float [128] sum_j dS_L S0 (PART 0), dbeta [64] (PART 1)
  static constexpr uint32_t EXTRA = DD + 512;             // float [128] dGam_63 extras (PART 0)
  static constexpr uint32_t BAR = EXTRA + 512;            // MMA done
  static constexpr uint32_t TBAR = BAR + 8;               // inputs landed
  static constexpr uint32_t CBAR = BAR + 16;              // [-dU; dO] landed (PART 0); dT, placed dP (PART 1)
  static constexpr uint32_t SBAR = BAR + 24;              // S0 (BF16 tile) landed (PART 0)
  static constexpr uint32_t RBAR = BAR + 32;              // raw q and k tiles landed (PART 0)
  static constexpr uint32_t TMEM_SLOT = BAR + 40;
  static constexpr uint32_t TOTAL = BAR + 48;
  // PART 0 final partials (after the last MMAs): float [64][128] each
  static constexpr uint32_t PKM = GA, PDG = RU;
  // PART 1 final partials: float [64][128] and [32][128]
  static constexpr uint32_t QDG = XA, KMC = YA;
  // Store slabs, 4 KB per warp: PART 0 over dS_L (read only by products that
  // are done when dv and the final epilogue write), PART 1 over T, (I+M)^-1,
  // Y1 and dT (consumed; the next item's copies are issued after the final
  // epilogue).
  static constexpr uint32_t SLAB0 = DST, SLAB1 = TT;
  // PART 0: the raw q and k tiles [64 tok][128 ch] for the final epilogue, in
  // space only the Gram part uses (its gate factors, G, and its Ai, Y1, dT tiles).
  static constexpr uint32_t RAWQ = 168960, RAWK = AIT;
  static_assert(GG + 17408 <= TT && MT + 4224 <= GG, "G");
  static_assert(YS + 2048 <= ZS && DST + 32768 <= YS, "scan scratch clears dS_L");
  static_assert(GB + 24576 <= RU + 32768 && RU + 32768 <= GST, "[R; U] stays clear of Gam");
  static_assert(CST + 6144 <= XM + 17408 && ZS + 6144 <= GG, "gate factors");
  static_assert(TOTAL + 1024 <= 232448, "shared memory");
  static_assert(SLAB0 + 32768 <= YS && (SLAB0 >= PDG + 32768 || SLAB0 + 32768 <= PKM) &&
                    (SLAB0 >= BT2 + 32768 || SLAB0 + 32768 <= BT2), "PART 0 slabs clear of the live partials and scan scratch");
  static_assert(RAWQ >= YS + 2048 && RAWQ + 16384 <= TT && RAWK + 16384 <= BETA && RAWQ % 1024 == 0 &&
                    RAWK % 1024 == 0, "PART 0 raw q, k tiles: clear of the scan scratch, T and beta; swizzle alignment");
  static_assert(SLAB1 >= KMC + 32768 && SLAB1 >= GG + 17408 && SLAB1 + 32768 <= BETA,
                "PART 1 slabs clear of the partials, G and beta");
};

// FP32 [64 tokens][128 channels] arrays read both with one token per lane
// (float4 groups of channels) and with one channel per thread: the float4
// slot of channels 4f..4f+3 of token r is XOR-ed with the token's low five
// bits, so a warp reading one group of 32 tokens, or one token's channels,
// touches every bank.
__device__ __forceinline__ int sw4(int r, int f) { return r * 32 + (f ^ (r & 31)); }
__device__ __forceinline__ int sw(int r, int ch) { return 4 * sw4(r, ch >> 2) + (ch & 3); }
__device__ __forceinline__ float4 f4mul(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
__device__ __forceinline__ float4 f4exp(float4 a) { return make_float4(__expf(a.x), __expf(a.y), __expf(a.z), __expf(a.w)); }

__device__ __forceinline__ void st_chunk_s(uint8_t *dst, const float *x) {
  *reinterpret_cast<uint4 *>(dst) = make_uint4(tc::pack_bf16(x[0], x[1]), tc::pack_bf16(x[2], x[3]),
                                               tc::pack_bf16(x[4], x[5]), tc::pack_bf16(x[6], x[7]));
}

// Gradient rows leave through a warp's 4 KB slab of shared memory.  Lane l
// holds token row l of a [32 rows][32 FP32 columns] block; it puts its eight
// float4 pieces into row l of the slab, piece j at slot j ^ (l & 7), and the
// block then leaves four whole 128-byte rows per warp instruction (lane l
// takes row 4i + (l >> 3), piece l & 7) instead of 32 rows of 16 bytes each.
// Both sides touch every bank once per quarter warp.
__device__ __forceinline__ void slab_put(float4 *slab, int lane, int j, float4 v) {
  slab[lane * 8 + (j ^ (lane & 7))] = v;
}
// Rows at or past `rows` are not written; ADD: FP32 reductions onto global memory.
template <bool ADD>
__device__ __forceinline__ void slab_rows_out(const float4 *slab, float *dst, size_t row_stride, int rows,
                                              int lane) {
  __syncwarp();
  const int j = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int R = 4 * i + (lane >> 3);
    const float4 v = slab[R * 8 + (j ^ (R & 7))];
    float4 *d = reinterpret_cast<float4 *>(dst + (size_t)R * row_stride) + j;
    if (R < rows) {
      if (ADD) atomicAdd(d, v);
      else *d = v;
    }
  }
  __syncwarp();   // every lane has read the slab before it is filled again
}

struct BwdItemArgs {
  const float *beta;
  const uint8_t *s0_init;      // BF16 state tiles [N*H] of the initial states, or null
  const uint8_t *s0_ck;        // BF16 state tiles at every full chunk end, [chunk][H]
  const int32_t *cu;
  const int64_t *pref;         // [N+1] chunks before sequence n
  const int64_t *prefck;       // [N+1] full chunks (stored states) before sequence n
  const uint8_t *dsl;          // dS_L per packet: BF16 [128 ch][128 v] tile
  const uint8_t *ndu;          // -dU per packet: BF16 [64 tok][128 v] tile
  const uint8_t *dot;          // dO per packet: BF16 [64 tok][128 v] tile
  uint8_t *dtp;                // per packet, from the state part to the Gram part (kDtpBytes):
                               //   dT as the BF16 [64][64] operand tile, rows 64..127 of the
                               //   [dG; dP] tile (dP placed, BF16, 2 x 8 KB), dP^T FP32 [64][64]
  const uint8_t *tt;           // T and (I + M)^-1 per packet from the forward: BF16 [64][64] tiles
  const ItemRec *items;        // where each packet sits (from the dO tile conversion)
  float *dq, *dk, *dv, *dg, *dbeta;
  int N, H;
  int32_t *dev_status;
  uint64_t wait_ns;
};

constexpr uint32_t kDtpBytes = 8192 + 16384 + 16384;

template <int PART>
__global__ void __launch_bounds__(kThreads, 1)
bwd_item_kernel(const __grid_constant__ TmaMaps maps, const BwdItemArgs a) {
  using Lay = BItemLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t *sp = smem_raw + (sb - sraw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hw = warp >> 2;
  const int H = a.H;

  float *s_beta = reinterpret_cast<float *>(sp + Lay::BETA);
  float *s_red = reinterpret_cast<float *>(sp + Lay::RED);
  // gate factors during the prep (the Gram part keeps YA's second block free for dP^T)
  float *s_cst = reinterpret_cast<float *>(sp + (PART == 0 ? Lay::CST : Lay::ZS));
  float *s_Y = reinterpret_cast<float *>(sp + Lay::YS);
  float *s_G = reinterpret_cast<float *>(sp + Lay::GG);
  float *s_gam = reinterpret_cast<float *>(sp + Lay::GST);
  float *s_dd = reinterpret_cast<float *>(sp + Lay::DD);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sp + Lay::BAR);
  uint64_t *tbar = reinterpret_cast<uint64_t *>(sp + Lay::TBAR);
  uint64_t *cbar = reinterpret_cast<uint64_t *>(sp + Lay::CBAR);
  uint64_t *s0bar = reinterpret_cast<uint64_t *>(sp + Lay::SBAR);
  uint64_t *rbar = reinterpret_cast<uint64_t *>(sp + Lay::RBAR);

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(tbar, 1);
    mbar_init(cbar, 1);
    mbar_init(s0bar, 1);
    mbar_init(rbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tc::tmem_alloc(sb + Lay::TMEM_SLOT, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + Lay::TMEM_SLOT);
  const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
  uint32_t phase = 0, tphase = 0, cphase = 0, s0phase = 0, rphase = 0;
  bool s0pend = false;   // an S0 copy is in flight (PART 0)
  bool rpend = false;    // raw q, k copies are in flight (PART 0)
  bool aborted = false;
  const int N = a.N;
  const int64_t total = a.pref[N] * H;

  // Item pp (sequence, head, chunk) in packet order: pp = H pref[n] + h c_n + j.
  auto locate = [&](int64_t pp, int &n_, int &h_, int64_t &j_, int64_t &t0_, int &L_) {
    const ItemRec rec = a.items[pp];
    n_ = rec.n;
    h_ = rec.h;
    j_ = rec.j;
    t0_ = rec.t0;
    L_ = rec.L;
  };
  // Inputs: g into its staging rows and beta (both parts), q, k into the Gram A
  // tile, v (the state part); with g, the item's T (and for the Gram part
  // (I + M)^-1) as the forward formed them.  `arrive`: this issue completes
  // the barrier phase's arrival (the other only adds its bytes).
  constexpr uint32_t kTtBytes = PART == 0 ? 8192 : 16384;
  constexpr uint32_t kGBytes = 32768 + kTtBytes;                 // g, T (, Ai)
  constexpr uint32_t kKqvBytes = PART == 0 ? 16384 + 16384 : 32768;   // k, v | k, q
  auto issue_g = [&](int h_, int64_t t0_, int L_, int64_t pp, bool arrive, uint32_t bytes) {
    if (tid == 32) {
      if (arrive) mbar_expect_tx(sb + Lay::TBAR, bytes);
      else mbar_add_tx(sb + Lay::TBAR, bytes);
      tma_load_3d(sb + Lay::GST, &maps.g, 0, h_, (int)t0_, sb + Lay::TBAR);
      bulk_load(sb + Lay::TT, a.tt + (size_t)pp * 16384, kTtBytes, sb + Lay::TBAR);
    }
    if (tid >= 64 && tid < 64 + kC) {
      const int r = tid - 64;
      const bool ok = r < L_;
      cp_async4(sb + Lay::BETA + 4 * r, a.beta + (ok ? (size_t)(t0_ + r) * H + h_ : 0), ok);
    }
    cp_async_commit();
  };
  auto issue_kqv = [&](int h_, int64_t t0_) {   // tid 32, after its expect_tx
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (PART == 1) {   // k and q into the rows of the Gram A tile their scaled versions replace
        tma_load_3d(sb + Lay::GA + b * 16384, &maps.k, 64 * b, h_, (int)t0_, sb + Lay::TBAR);
        tma_load_3d(sb + Lay::GA + b * 16384 + 8192, &maps.q, 64 * b, h_, (int)t0_, sb + Lay::TBAR);
      } else {           // k into the Ktilde tile, scaled in place by the prep
        tma_load_3d(sb + Lay::KT + b * 8192, &maps.k, 64 * b, h_, (int)t0_, sb + Lay::TBAR);
      }
      if (PART == 0) tma_load_3d(sb + Lay::VT + b * 8192, &maps.v, 64 * b, h_, (int)t0_, sb + Lay::TBAR);
    }
  };
  // Issued during the previous item's reverse scan: g and beta (state part),
  // all inputs (Gram part).
  bool pre = false;
  int n2 = 0, h2 = 0, L2 = 0;   // the next item, located while the current one's inputs land
  int64_t j2 = 0, t02 = 0;
  if ((int64_t)blockIdx.x < total) locate(blockIdx.x, n2, h2, j2, t02, L2);

  for (int64_t p = blockIdx.x; p < total && !aborted; p += gridDim.x) {
  const int n = n2, h = h2, L = L2;
  const int64_t j = j2, t0 = t02;
  const int unit = n * H + h;
  const int64_t ckb = a.prefck[n];

  if (PART == 1 && !pre) {
    issue_g(h, t0, L, p, true, kGBytes + kKqvBytes);
    if (tid == 32) issue_kqv(h, t0);
  }
  if (PART == 0) {
    if (!pre) issue_g(h, t0, L, p, false, kGBytes);
    if (tid == 32) {
      mbar_expect_tx(sb + Lay::TBAR, kKqvBytes);
      issue_kqv(h, t0);
      // The raw q and k tiles, read only by the final epilogue.
      mbar_expect_tx(sb + Lay::RBAR, 32768);
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        tma_load_3d(sb + Lay::RAWQ + b * 8192, &maps.q, 64 * b, h, (int)t0, sb + Lay::RBAR);
        tma_load_3d(sb + Lay::RAWK + b * 8192, &maps.k, 64 * b, h, (int)t0, sb + Lay::RBAR);
      }
    }
    rpend = true;
  }
  pre = false;
  const bool has_next = p + gridDim.x < total;
  if (has_next) locate(p + gridDim.x, n2, h2, j2, t02, L2);
  // The per-chunk states and gradients come from L2 later; start them now.
  const uint8_t *S0src = j == 0 ? (a.s0_init ? a.s0_init + (size_t)unit * 32768 : nullptr)
                                : a.s0_ck + ((size_t)(ckb + j - 1) * H + h) * 32768;
  // The state part takes T from the forward and needs no Gram tiles: S0 (the
  // BF16 operand tile) lands in the Gram A tile's space from the start.
  if (PART == 0 && S0src) {
    s0pend = true;
    if (tid == 32) {
      mbar_expect_tx(sb + Lay::SBAR, 32768);
      bulk_load(sb + Lay::S0T, S0src, 32768, sb + Lay::SBAR);
    }
  }
  if (PART == 1 && tid == 32) {   // dT's operand tile and the placed dP rows of [dG; dP]
    const uint8_t *dt = a.dtp + (size_t)p * kDtpBytes;
    mbar_expect_tx(sb + Lay::CBAR, 40960);
    bulk_load(sb + Lay::DTT, dt, 8192, sb + Lay::CBAR);
    bulk_load(sb + Lay::XA + 8192, dt + 8192, 8192, sb + Lay::CBAR);
    bulk_load(sb + Lay::XA + 16384 + 8192, dt + 16384, 8192, sb + Lay::CBAR);
    bulk_load(sb + Lay::YA + 16384, dt + 24576, 16384, sb + Lay::CBAR);   // dP^T (FP32) where its tile goes
  }

  cp_async_wait_all();
  if (__syncthreads_or(!wait_timed(tbar, tphase, a.wait_ns))) aborted = true;
  tphase ^= 1;

  // ---------------- gate prep ----------------
  // Warp w owns rows 8w..8w+7 (half hf = w / 4), lane l owns channels 4l..4l+3.
  if (!aborted) {
    const int hf = warp >> 2, cq = lane >> 1, sub = (lane & 1) * 8;
    float2 gm[8][2];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 8 * warp + i;
      const float4 x = r < L ? *reinterpret_cast<const float4 *>(sp + Lay::GST + r * 512 + lane * 16)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      gm[i][0] = make_float2(x.x, x.y);
      gm[i][1] = make_float2(x.z, x.w);
    }
#pragma unroll
    for (int i = 1; i < 8; ++i)
#pragma unroll
      for (int c = 0; c < 2; ++c) gm[i][c] = __fadd2_rn(gm[i][c], gm[i - 1][c]);
    *reinterpret_cast<float4 *>(s_red + warp * 128 + 4 * lane) =
        make_float4(gm[7][0].x, gm[7][0].y, gm[7][1].x, gm[7][1].y);
    __syncthreads();
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
      // Slots per half: -ref, fk, fk2, fh, fh2, cb (as in the forward's prep).
      float f[12];
      f[0] = -G15; f[1] = 1.f; f[2] = __expf(G15);
      f[3] = __expf(G31 - G15); f[4] = __expf(G63 - G31); f[5] = __expf(G47 - G15);
      f[6] = -G47; f[7] = __expf(G47 - G31); f[8] = __expf(G31);
      f[9] = __expf(G63 - G47); f[10] = 1.f; f[11] = 0.f;
#pragma unroll
      for (int q2 = 0; q2 < 12; ++q2) s_cst[q2 * 128 + ch] = f[q2];
    }
    __syncthreads();
    float2 nref[2], fk[2], fk2[2], cb[2];
    {
      auto ld4 = [&](int slot, float2 *d) {
        const float4 x = *reinterpret_cast<const float4 *>(s_cst + (hf * 6 + slot) * 128 + 4 * lane);
        d[0] = make_float2(x.x, x.y);
        d[1] = make_float2(x.z, x.w);
      };
      float2 base[2];
      const float4 bv = *reinterpret_cast<const float4 *>(s_red + warp * 128 + 4 * lane);
      base[0] = make_float2(bv.x, bv.y);
      base[1] = make_float2(bv.z, bv.w);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 2; ++c) gm[i][c] = __fadd2_rn(gm[i][c], base[c]);
      ld4(0, nref); ld4(1, fk); ld4(2, fk2); ld4(5, cb);
    }
    auto st4 = [&](uint8_t *dst, const float2 *x) {
      *reinterpret_cast<uint2 *>(dst) = make_uint2(tc::pack_bf16(x[0].x, x[0].y), tc::pack_bf16(x[1].x, x[1].y));
    };
    auto un4 = [&](const uint2 &u, float2 *x) {
      x[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
      x[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    };
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 8 * warp + i;
      float2 kk[2], qq[2], x[2], y[2], t[2];
      {
        const bool in = r < L;
        const uint2 z2 = make_uint2(0, 0);
        const uint2 kv = !in ? z2
                         : PART == 1 ? *reinterpret_cast<const uint2 *>(sp + Lay::GA + tc::tile_offset(128, r, cq) + sub)
                                     : *reinterpret_cast<const uint2 *>(sp + Lay::KT + tc::tile_offset(64, r, cq) + sub);
        un4(kv, kk);
        if (PART == 1) {
          const uint2 qv = in ? *reinterpret_cast<const uint2 *>(sp + Lay::GA + tc::tile_offset(128, 64 + r, cq) + sub) : z2;
          un4(qv, qq);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float2 d = __fadd2_rn(gm[i][c], nref[c]);
        x[c] = make_float2(__expf(d.x), __expf(d.y));   // exp(Gam_r - ref), within [e^-80, e^80]
        if (PART == 1) y[c] = make_float2(__expf(-d.x), __expf(-d.y)); // exp(ref - Gam_r)
      }
      if (PART == 1) {   // the gated Gram operands (the state part takes T from the forward)
#pragma unroll
        for (int c = 0; c < 2; ++c) t[c] = __fmul2_rn(kk[c], x[c]);
        st4(sp + Lay::GA + tc::tile_offset(128, r, cq) + sub, t);
#pragma unroll
        for (int c = 0; c < 2; ++c) t[c] = __fmul2_rn(qq[c], x[c]);
        st4(sp + Lay::GA + tc::tile_offset(128, 64 + r, cq) + sub, t);
#pragma unroll
        for (int c = 0; c < 2; ++c) t[c] = __fmul2_rn(kk[c], y[c]);
        st4(sp + Lay::GB + tc::tile_offset(96, hf ? 32 + r : r, cq) + sub, t);
        if (!hf) {
#pragma unroll
          for (int c = 0; c < 2; ++c) t[c] = __fmul2_rn(kk[c], __fmul2_rn(y[c], cb[c]));
          st4(sp + Lay::GB + tc::tile_offset(96, 32 + r, cq) + sub, t);
        }
      }
      if (PART == 0) {   // Ktilde = k exp(Gam_r) = k (x fk) fk2
#pragma unroll
        for (int c = 0; c < 2; ++c) t[c] = __fmul2_rn(kk[c], __fmul2_rn(__fmul2_rn(x[c], fk[c]), fk2[c]));
        st4(sp + Lay::KT + tc::tile_offset(64, r, cq) + sub, t);
      }
    }
    // Gam stays for the final epilogue, in place of g (every thread has read
    // its g rows before the first barrier of the prep).
#pragma unroll
    for (int i = 0; i < 8; ++i)
      reinterpret_cast<float4 *>(s_gam)[sw4(8 * warp + i, lane)] =
          make_float4(gm[i][0].x, gm[i][0].y, gm[i][1].x, gm[i][1].y);
    tc::fence_smem_to_async();
    __syncthreads();
  }

  // ---------------- the Gram part: gated Gram products, one [128 x 96 x 128] MMA ----------------
  // (T and (I + M)^-1 come from the forward, so only G is read back.)
  if (PART == 1) {
    if (!aborted && tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 96, 0, 0);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem, tc::desc_kmajor(sb + Lay::GA, 128, s2), tc::desc_kmajor(sb + Lay::GB, 96, s2),
                     id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (!aborted && __syncthreads_or(!wait_timed(bar, phase, a.wait_ns))) aborted = true;
    phase ^= 1;
    tc::fence_after_sync();
    // Gram rows (lane m = row m, k rows only): G, strictly lower.
    if (!aborted) {
      const int m = 32 * qd + lane, part = m >> 6, r = m & 63, second = r >> 5;
      const int i0 = second ? 32 * hw : (hw ? 32 : 0);
      float acc[32];
      if (second || hw == 0) {
        tc::tmem_ld32(tl + (second ? 32 + 32 * hw : 0), acc);
        tc::tmem_wait_ld();
      }
      const bool zero = !second && hw;
      if (part == 0) {
        float4 *gdst = reinterpret_cast<float4 *>(s_G + r * 68 + i0);
        auto gv = [&](int jj) { return (!zero && i0 + jj < r) ? acc[jj] : 0.f; };
#pragma unroll
        for (int jj = 0; jj < 32; jj += 4) gdst[jj >> 2] = make_float4(gv(jj), gv(jj + 1), gv(jj + 2), gv(jj + 3));
      }
    }
    tc::fence_before_sync();
    __syncthreads();
  }
  const size_t row_stride = (size_t)H * kD;   // elements between tokens in [T][H][128]
  const size_t base_row = ((size_t)t0 * H + h) * kD;
  if constexpr (PART == 0) {
    // ---- S0 as the BF16 [ch][v] tile: copied in, or zero without an initial state ----
    if (!aborted) {
      if (S0src) {
        if (__syncthreads_or(!wait_timed(s0bar, s0phase, a.wait_ns))) {
          aborted = true;
        } else {
          s0pend = false;
          s0phase ^= 1;
        }
      } else {
        for (int e = tid; e < 2048; e += kThreads)
          reinterpret_cast<uint4 *>(sp + Lay::S0T)[e] = make_uint4(0, 0, 0, 0);
        tc::fence_smem_to_async();
        __syncthreads();
      }
    }
    // ---- R = V - Ktilde S0 (TMEM columns 128..255) ----
    if (!aborted && tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem + 128, tc::desc_kmajor(sb + Lay::KT, 64, s2),
                     tc::desc_mnmajor(sb + Lay::S0T, 128, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (!aborted && __syncthreads_or(!wait_timed(bar, phase, a.wait_ns))) aborted = true;
    phase ^= 1;
    tc::fence_after_sync();
    if (!aborted && qd < 2) {   // rows 64..127 of [U; R]; V rows past the chunk's end are zero
      const int r = 32 * qd + lane;
      float acc[64];
      tc::tmem_ld32(tl + 128 + hw * 64, *reinterpret_cast<float(*)[32]>(acc));
      tc::tmem_ld32(tl + 128 + hw * 64 + 32, *reinterpret_cast<float(*)[32]>(acc + 32));
      tc::tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const int chunk = hw * 8 + cc;
        float xv[8];
        unpack8(*reinterpret_cast<const uint4 *>(sp + Lay::VT + tc::tile_offset(64, r, chunk)), xv);
#pragma unroll
        for (int e = 0; e < 8; ++e) xv[e] = (r < L ? xv[e] : 0.f) - acc[8 * cc + e];
        st_chunk_s(sp + Lay::RU + tc::tile_offset(128, 64 + r, chunk), xv);
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    // ---- U = T R (columns 256..383); the chain's [-dU; dO] tile lands over Ktilde, V ----
    // [-dU; dO] lands over Ktilde and V as one 128-row tile (each 64-row
    // tile's column blocks interleaved), dS_L over the consumed M, (I+M)^-1.
    if (!aborted && tid == 32) {
      mbar_expect_tx(sb + Lay::CBAR, 65536);
      const uint8_t *nd = a.ndu + (size_t)p * 16384, *dd = a.dot + (size_t)p * 16384;
      bulk_load(sb + Lay::BT2, nd, 8192, sb + Lay::CBAR);
      bulk_load(sb + Lay::BT2 + 16384, nd + 8192, 8192, sb + Lay::CBAR);
      bulk_load(sb + Lay::BT2 + 8192, dd, 8192, sb + Lay::CBAR);
      bulk_load(sb + Lay::BT2 + 24576, dd + 8192, 8192, sb + Lay::CBAR);
      bulk_load(sb + Lay::DST, a.dsl + (size_t)p * 32768, 32768, sb + Lay::CBAR);
    }
    if (!aborted && tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + 256, tc::desc_kmajor(sb + Lay::TT, 64, s2),
                     tc::desc_mnmajor(sb + Lay::RU + 8192, 128, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (!aborted && __syncthreads_or(!wait_timed(bar, phase, a.wait_ns))) aborted = true;
    phase ^= 1;
    tc::fence_after_sync();
    if (!aborted && qd < 2) {   // rows 0..63 of [U; R]
      const int r = 32 * qd + lane;
      float acc[64];
      tc::tmem_ld32(tl + 256 + hw * 64, *reinterpret_cast<float(*)[32]>(acc));
      tc::tmem_ld32(tl + 256 + hw * 64 + 32, *reinterpret_cast<float(*)[32]>(acc + 32));
      tc::tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        st_chunk_s(sp + Lay::RU + tc::tile_offset(128, r, hw * 8 + cc), acc + 8 * cc);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    if (!aborted && __syncthreads_or(!wait_timed(cbar, cphase, a.wait_ns))) aborted = true;
    cphase ^= 1;
    // ---- dR = T^T (-dU) -> -dR (columns 0..127);  [-dU; dO] [U; R]^T (384..511):
    //      rows 0..63 x 64..127 = -dT, rows 64..127 x 0..63 = dP;  [U; R] dS_L^T (256..383):
    //      rows 0..63 = dKhat ----
    if (!aborted && tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t idr = tc::idesc_bf16(128, 128, 1, 1);
      constexpr uint32_t idk = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + 0, tc::desc_mnmajor(sb + Lay::TT, 64, s2),
                     tc::desc_mnmajor(sb + Lay::BT2, 128, s2), idr, s2 > 0);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem + 384, tc::desc_kmajor(sb + Lay::BT2, 128, s2),
                     tc::desc_kmajor(sb + Lay::RU, 128, s2), idk, s2 > 0);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem + 256, tc::desc_kmajor(sb + Lay::RU, 128, s2),
                     tc::desc_kmajor(sb + Lay::DST, 128, s2), idk, s2 > 0);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)   // dS_L S0^T: its diagonal is dd_c = sum_v dS_L[c, v] S0[c, v]
        tc::mma_bf16(tmem + 128, tc::desc_kmajor(sb + Lay::DST, 128, s2),
                     tc::desc_kmajor(sb + Lay::S0T, 128, s2), idk, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (!aborted && __syncthreads_or(!wait_timed(bar, phase, a.wait_ns))) aborted = true;
    phase ^= 1;
    tc::fence_after_sync();
    uint8_t *dtp = a.dtp + (size_t)p * kDtpBytes;
    if (!aborted && hw == 0) {   // the diagonal of dS_L S0^T: lane c takes column c
      float x[32];
      tc::tmem_ld32(tl + 128 + 32 * qd, x);
      tc::tmem_wait_ld();
      float dd = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) dd = e == lane ? x[e] : dd;
      s_dd[32 * qd + lane] = dd;
    }
    if (!aborted) {
      if (qd < 2) {   // -dR replaces -dU in rows 0..63: the next product's operand first
        const int r = 32 * qd + lane;
        float acc[64];
        tc::tmem_ld32(tl + 0 + hw * 64, *reinterpret_cast<float(*)[32]>(acc));
        tc::tmem_ld32(tl + 0 + hw * 64 + 32, *reinterpret_cast<float(*)[32]>(acc + 32));
        tc::tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          st_chunk_s(sp + Lay::BT2 + tc::tile_offset(128, r, hw * 8 + cc), acc + 8 * cc);
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    // ---- [dKtilde; dQtilde] = [-dR; dO] S0^T (columns 128..255) ----
    if (!aborted && tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem + 128, tc::desc_kmajor(sb + Lay::BT2, 128, s2),
                     tc::desc_kmajor(sb + Lay::S0T, 128, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    // While the product runs: dv (= dR), dT and dP leave for global memory
    // (their TMEM columns are not the product's).
    if (!aborted && qd < 2) {
      const int r = 32 * qd + lane;
      float4 *slab = reinterpret_cast<float4 *>(sp + Lay::SLAB0) + warp * 256;
      float *dst = a.dv + base_row + (size_t)(32 * qd) * row_stride + hw * 64;
#pragma unroll
      for (int half = 0; half < 2; ++half) {   // warp-wide TMEM loads; stores for tokens inside the chunk
        float acc[32];
        tc::tmem_ld32(tl + 0 + hw * 64 + 32 * half, acc);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          slab_put(slab, lane, e >> 2, make_float4(-acc[e], -acc[e + 1], -acc[e + 2], -acc[e + 3]));
        slab_rows_out<false>(slab, dst + 32 * half, row_stride, L - 32 * qd, lane);
      }
      float d2[32];   // dT row r, columns 32 hw .. +31 (kept on and below the diagonal)
      tc::tmem_ld32(tl + 448 + hw * 32, d2);
      tc::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) d2[e] = 32 * hw + e <= r ? -d2[e] : 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {   // the Gram part's dT operand tile
        const float *x = d2 + 8 * cc;
        *reinterpret_cast<uint4 *>(dtp + tc::tile_offset(64, r, 4 * hw + cc)) =
            make_uint4(tc::pack_bf16(x[0], x[1]), tc::pack_bf16(x[2], x[3]),
                       tc::pack_bf16(x[4], x[5]), tc::pack_bf16(x[6], x[7]));
      }
    } else if (!aborted) {
      // dP row r, columns i = 32 hw .. +31 (i <= r): placed against Gram B as
      // rows 64..127 of [dG; dP] (first-half rows at kappa = i, second-half rows
      // at kappa = 32 + i, zeros elsewhere; K = 96), and transposed (FP32) for
      // the placement against Gram A.
      const int r = 32 * (qd - 2) + lane;
      float d2[32];
      tc::tmem_ld32(tl + 384 + hw * 32, d2);
      tc::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) d2[e] = 32 * hw + e <= r ? d2[e] : 0.f;
      uint8_t *xa = dtp + 8192;   // [2 blocks][rows 64..127][128 B]
      auto put = [&](int ch, const float *x) {
        *reinterpret_cast<uint4 *>(xa + (ch >> 3) * 8192 + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) =
            make_uint4(tc::pack_bf16(x[0], x[1]), tc::pack_bf16(x[2], x[3]),
                       tc::pack_bf16(x[4], x[5]), tc::pack_bf16(x[6], x[7]));
      };
      const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (hw == 0) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          put((r < 32 ? 0 : 4) + cc, d2 + 8 * cc);
          put((r < 32 ? 4 : 0) + cc, z);
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) put(8 + cc, d2 + 8 * cc);
      }
      // dP^T row i (64 floats): float4 slot f stored at f ^ (i & 15), so that the
      // Gram part's reads of one slot of 16 consecutive rows spread over the banks
      float *dpt = reinterpret_cast<float *>(dtp + 24576);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int i = 32 * hw + e;
        dpt[i * 64 + ((((r >> 2) ^ (i & 15))) << 2) + (r & 3)] = d2[e];
      }
    }
    if (!aborted && __syncthreads_or(!wait_timed(bar, phase, a.wait_ns))) aborted = true;
    phase ^= 1;
    tc::fence_after_sync();
    if (!aborted) {
      if (__syncthreads_or(!wait_timed(rbar, rphase, a.wait_ns))) {
        aborted = true;
      } else {
        rpend = false;
        rphase ^= 1;
      }
    }
    // ---- final epilogue: dq, dk and dGam from Qtilde, Ktilde, Khat and d ----
    // Token r's dQtilde sits in TMEM lane 64 + r, its dKtilde and dKhat in lane
    // r: the two halves of the CTA work at once, each on its own dGam part.
    float4 *pdq4 = reinterpret_cast<float4 *>(sp + Lay::PKM);   // q (dq from Qtilde)
    float4 *pdk4 = reinterpret_cast<float4 *>(sp + Lay::PDG);   // k (dk+ - dk-)
    float4 *pkk4 = reinterpret_cast<float4 *>(sp + Lay::BT2);   // k (dk from Khat): the dGam_63 extra
    const float4 *g4 = reinterpret_cast<const float4 *>(s_gam);
    float4 *slab = reinterpret_cast<float4 *>(sp + Lay::SLAB0) + warp * 256;
    if (!aborted && qd >= 2) {
      const int r = 32 * (qd - 2) + lane;
      float aq[64];
      tc::tmem_ld32(tl + 128 + hw * 64, *reinterpret_cast<float(*)[32]>(aq));
      tc::tmem_ld32(tl + 128 + hw * 64 + 32, *reinterpret_cast<float(*)[32]>(aq + 32));
      tc::tmem_wait_ld();
      float *dst = a.dq + base_row + (size_t)(32 * (qd - 2)) * row_stride + hw * 64;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int u = 4 * half; u < 4 * half + 4; ++u) {
          float qv[8];   // raw q of token r (zero past the chunk's end)
          unpack8(r < L ? *reinterpret_cast<const uint4 *>(sp + Lay::RAWQ + tc::tile_offset(64, r, hw * 8 + u))
                        : make_uint4(0, 0, 0, 0), qv);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {   // channels hw*64 + 8u + 4hf .. +3
            const int F = hw * 16 + 2 * u + hf, c = 8 * u + 4 * hf;
            const float4 dqa = f4mul(f4exp(g4[sw4(r, F)]), make_float4(aq[c], aq[c + 1], aq[c + 2], aq[c + 3]));
            pdq4[sw4(r, F)] = f4mul(make_float4(qv[4 * hf], qv[4 * hf + 1], qv[4 * hf + 2], qv[4 * hf + 3]), dqa);
            slab_put(slab, lane, (2 * u + hf) & 7, dqa);
          }
        }
        slab_rows_out<false>(slab, dst + 32 * half, row_stride, L - 32 * (qd - 2), lane);
      }
    } else if (!aborted) {
      const int r = 32 * qd + lane;
      float ak[64], ah[64];
      tc::tmem_ld32(tl + 128 + hw * 64, *reinterpret_cast<float(*)[32]>(ak));
      tc::tmem_ld32(tl + 128 + hw * 64 + 32, *reinterpret_cast<float(*)[32]>(ak + 32));
      tc::tmem_ld32(tl + 256 + hw * 64, *reinterpret_cast<float(*)[32]>(ah));
      tc::tmem_ld32(tl + 256 + hw * 64 + 32, *reinterpret_cast<float(*)[32]>(ah + 32));
      tc::tmem_wait_ld();
      float *dst = a.dk + base_row + (size_t)(32 * qd) * row_stride + hw * 64;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int u = 4 * half; u < 4 * half + 4; ++u) {
          float kv[8];   // raw k of token r (zero past the chunk's end)
          unpack8(r < L ? *reinterpret_cast<const uint4 *>(sp + Lay::RAWK + tc::tile_offset(64, r, hw * 8 + u))
                        : make_uint4(0, 0, 0, 0), kv);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int F = hw * 16 + 2 * u + hf, c = 8 * u + 4 * hf;
            const float4 gam = g4[sw4(r, F)], g63 = g4[sw4(63, F)];
            const float4 dkp = f4mul(f4exp(gam), make_float4(ak[c], ak[c + 1], ak[c + 2], ak[c + 3]));
            const float4 dkm = f4mul(f4exp(make_float4(g63.x - gam.x, g63.y - gam.y, g63.z - gam.z, g63.w - gam.w)),
                                     make_float4(ah[c], ah[c + 1], ah[c + 2], ah[c + 3]));
            const float4 k4 = make_float4(kv[4 * hf], kv[4 * hf + 1], kv[4 * hf + 2], kv[4 * hf + 3]);
            const float4 kp = f4mul(k4, dkp), km = f4mul(k4, dkm);
            pdk4[sw4(r, F)] = make_float4(kp.x - km.x, kp.y - km.y, kp.z - km.z, kp.w - km.w);
            pkk4[sw4(r, F)] = km;
            slab_put(slab, lane, (2 * u + hf) & 7, make_float4(dkp.x + dkm.x, dkp.y + dkm.y, dkp.z + dkm.z, dkp.w + dkm.w));
          }
        }
        slab_rows_out<false>(slab, dst + 32 * half, row_stride, L - 32 * qd, lane);
      }
    }
    // Gam leaves its rows for the next item's g; the scan keeps exp(Gam_63).
    const float e63 = tid < 128 ? __expf(s_gam[sw(63, tid)]) : 0.f;
    tc::fence_smem_to_async();
    __syncthreads();
    if (!aborted && has_next) {
      issue_g(h2, t02, L2, p + gridDim.x, false, kGBytes);
      pre = true;
    }
    // dg = reverse cumulative sum of dGam plus the Gam_63 terms (sum_r k dk-_r from
    // Khat, d * sum_v dS_L S0).  Two threads per channel, 32 rows each.
    float *sred = s_Y;   // [2][128] partial sums, [2][128] partial extras
    if (!aborted) {
      const int ch = tid & 127, hf = tid >> 7;
      const float *pdq = reinterpret_cast<const float *>(pdq4), *pdk = reinterpret_cast<const float *>(pdk4);
      const float *pkk = reinterpret_cast<const float *>(pkk4);
      float dgam[32], part = 0.f, extra = 0.f;   // dGam of rows 32 hf + i, kept for the suffix sums
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = 32 * hf + i;
        dgam[i] = pdq[sw(r, ch)] + pdk[sw(r, ch)];
        part += dgam[i];
        extra += pkk[sw(r, ch)];
      }
      if (hf == 0) extra = fmaf(e63, s_dd[ch], extra);
      sred[hf * 128 + ch] = part;
      sred[256 + hf * 128 + ch] = extra;
      __syncthreads();
      float suffix = sred[256 + ch] + sred[384 + ch] + (hf == 0 ? sred[128 + ch] : 0.f);
#pragma unroll
      for (int i = 31; i >= 0; --i) {
        const int r = 32 * hf + i;
        suffix += dgam[i];
        if (r < L) a.dg[base_row + (size_t)r * row_stride + ch] = suffix;
      }
    }
  } else {
    // ---- PART 1: dT (its operand tile) and dP from the state part ----
    const float *dPT = reinterpret_cast<const float *>(sp + Lay::YA + 16384);   // FP32 [64][64], copied in
    float *s_db = s_dd;   // dbeta [64]
    if (!aborted && __syncthreads_or(!wait_timed(cbar, cphase, a.wait_ns))) aborted = true;
    cphase ^= 1;
    // ---- Y1 = Ai^T dT (columns 128..191) ----
    if (!aborted && tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 64, 1, 1);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + 128, tc::desc_mnmajor(sb + Lay::AIT, 64, s2),
                     tc::desc_mnmajor(sb + Lay::DTT, 64, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (!aborted && __syncthreads_or(!wait_timed(bar, phase, a.wait_ns))) aborted = true;
    phase ^= 1;
    tc::fence_after_sync();
    if (!aborted && qd < 2) {   // dbeta_j = Y1_jj (the T part); Y1 as a K-major operand
      const int jr = 32 * qd + lane;
      float y[32];
      tc::tmem_ld32(tl + 128 + hw * 32, y);
      tc::tmem_wait_ld();
      if ((jr >> 5) == hw) {
        float dgl = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) dgl = e == (jr & 31) ? y[e] : dgl;
        s_db[jr] = dgl;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) st_chunk_s(sp + Lay::Y1T + tc::tile_offset(64, jr, hw * 4 + cc), y + 8 * cc);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    // ---- dA = -Y1 T^T (columns 256..319) and its transpose (384..447) ----
    if (!aborted && tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + 256, tc::desc_kmajor(sb + Lay::Y1T, 64, s2),
                     tc::desc_kmajor(sb + Lay::TT, 64, s2), id, s2 > 0);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + 384, tc::desc_kmajor(sb + Lay::TT, 64, s2),
                     tc::desc_kmajor(sb + Lay::Y1T, 64, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    // While they run: dP into columns 64..127 of YA (against the q x rows of
    // Gram A; rows 64..127 of XA came placed from the state part).  YA row i
    // (second index, own reference): dP_ri for r in i's half; row 64 + i (i in
    // the first half, second-half reference): dP_ri for r in the second half;
    // rows 96..127 zero.
    if (!aborted) {   // read every FP32 value, then write the tile over them
      const int m = tid >> 1, rh = (tid & 1) * 32;   // YA row m, P columns r = rh..rh+31
      float xv[32];
      const int src = m < 64 ? m : (m < 96 ? m - 64 : 0);
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const int f = (rh + e) >> 2;   // float4 slot of columns r = rh + e .. +3, stored at f ^ (src & 15)
        const float4 v4 = m < 96 ? *reinterpret_cast<const float4 *>(dPT + src * 64 + ((f ^ (src & 15)) << 2))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        xv[e] = v4.x; xv[e + 1] = v4.y; xv[e + 2] = v4.z; xv[e + 3] = v4.w;
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int r = rh + e;
        const bool keep = m < 64 ? ((m >> 5) == (r >> 5) && r >= m) : (m < 96 && r >= 32);
        xv[e] = keep ? xv[e] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        st_chunk_s(sp + Lay::YA + tc::tile_offset(128, m, 8 + (rh >> 3) + cc), xv + 8 * cc);
    }
    if (!aborted && __syncthreads_or(!wait_timed(bar, phase, a.wait_ns))) aborted = true;
    phase ^= 1;
    tc::fence_after_sync();
    if (!aborted) {
      if (qd < 2) {   // row rho of dA: dM, dbeta (the M part), dG into rows 0..63 of XA
        const int rho = 32 * qd + lane;
        float x[32];
        tc::tmem_ld32(tl + 256 + hw * 32, x);
        tc::tmem_wait_ld();
        const float br = s_beta[rho];
        float db = 0.f, vals[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int sig = 32 * hw + e;
          const float dm = sig < rho ? -x[e] : 0.f;
          db = fmaf(dm, s_G[rho * 68 + sig], db);
          vals[e] = br * dm;
        }
        atomicAdd(&s_db[rho], db);
        const int kbase = (rho < 32 ? 0 : 32) + 32 * hw;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_chunk_s(sp + Lay::XA + tc::tile_offset(128, rho, (kbase >> 3) + cc), vals + 8 * cc);
        if ((rho < 32) == (hw == 1)) {   // the four chunks of kappa this row leaves zero
          float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          const int kz = rho < 32 ? 64 : 0;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) st_chunk_s(sp + Lay::XA + tc::tile_offset(128, rho, (kz >> 3) + cc), z);
        }
        // Column sig = rho of dA, from the transposed product (its A operand has
        // 64 rows, so it too lands in TMEM lanes 0..63): dG^T into YA.
        const int sig = rho;
        tc::tmem_ld32(tl + 384 + hw * 32, x);
        tc::tmem_wait_ld();
        float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int r2 = 32 * hw + e;
          vals[e] = r2 > sig ? s_beta[r2] * (-x[e]) : 0.f;
        }
        const bool cross = sig < 32 && hw == 1;   // second-half rows against a first-half sig
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          st_chunk_s(sp + Lay::YA + tc::tile_offset(128, sig, hw * 4 + cc), cross ? z : vals + 8 * cc);
          st_chunk_s(sp + Lay::YA + tc::tile_offset(128, 64 + sig, hw * 4 + cc), cross ? vals + 8 * cc : z);
        }
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    // ---- [X; Xq] = [dG; dP] Gram B (columns 0..127), Y = [dG^T | dP^T] Gram A (128..255),
    //      whose lanes 64..95 hold the cross rows (first-half keys, second-half reference) ----
    if (!aborted && tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int s2 = 0; s2 < 6; ++s2)
        tc::mma_bf16(tmem + 0, tc::desc_kmajor(sb + Lay::XA, 128, s2),
                     tc::desc_mnmajor(sb + Lay::GB, 96, s2), id, s2 > 0);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem + 128, tc::desc_kmajor(sb + Lay::YA, 128, s2),
                     tc::desc_mnmajor(sb + Lay::GA, 128, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (!aborted && __syncthreads_or(!wait_timed(bar, phase, a.wait_ns))) aborted = true;
    phase ^= 1;
    tc::fence_after_sync();
    // ---- final epilogue: the rest of dq, dk, dGam; dbeta ----
    // dGam takes each gated pair's two sides from the very BF16 operands the
    // products used (Gram A rows for the sides where Gam enters with a plus
    // sign, Gram B rows for the others), so that the pair's terms, which the
    // reverse cumulative sum below sets against each other, cancel to FP32
    // accumulation precision.  Lanes 64..127 (Xq, and in lanes 64..95 the
    // cross rows of Y) and lanes 0..63 (X, Y) work at once, each half on its
    // own dGam part; the cross rows' terms of dk and dGam (keys 0..31) fall to
    // the warps of lanes 64..95, which have only dq otherwise, so that the
    // exponentials split evenly over the four lane quarters.  The parts of
    // dq, dk and dg go onto what the state part wrote as reductions in global
    // memory (no load, so no wait for the earlier values).
    float4 *qdg4 = reinterpret_cast<float4 *>(sp + Lay::QDG);   // dGam from the q side
    float4 *kdg4 = reinterpret_cast<float4 *>(sp + Lay::KMC);   // dGam from the k sides
    const float4 *g4 = reinterpret_cast<const float4 *>(s_gam);
    // 8 BF16 values of a tile row (one 16-byte chunk) as floats
    auto tile8 = [&](uint32_t tile, int rows, int row, int chunk, float *x) {
      unpack8(*reinterpret_cast<const uint4 *>(sp + tile + tc::tile_offset(rows, row, chunk)), x);
    };
    float *dqp = a.dq, *dkp_ = a.dk;
    float4 *slab = reinterpret_cast<float4 *>(sp + Lay::SLAB1) + warp * 256;
    if (!aborted && qd >= 2) {
      const int r = 32 * (qd - 2) + lane;
      const int ref = r < 32 ? 15 : 47;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int c0 = hw * 64 + 32 * half;
        const bool cross = qd == 2;   // key r < 32 also has a cross row (TMEM lane 64 + r of Y)
        float xq[32], yc[32];
        float4 km[8];
        tc::tmem_ld32(tl + 0 + c0, xq);
        if (cross) tc::tmem_ld32(tl + 128 + c0, yc);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 4; ++u) {   // 8 channels: one tile chunk
          float ga[8], gc[8];
          tile8(Lay::GA, 128, 64 + r, (c0 >> 3) + u, ga);
          if (cross) tile8(Lay::GB, 96, 32 + r, (c0 >> 3) + u, gc);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int F = (c0 >> 2) + 2 * u + hf, c = 8 * u + 4 * hf;
            const float4 gam = g4[sw4(r, F)], gref = g4[sw4(ref, F)];
            const float4 xqv = make_float4(xq[c], xq[c + 1], xq[c + 2], xq[c + 3]);
            const float4 add = f4mul(f4exp(make_float4(gam.x - gref.x, gam.y - gref.y, gam.z - gref.z, gam.w - gref.w)), xqv);
            float4 qa = f4mul(make_float4(ga[4 * hf], ga[4 * hf + 1], ga[4 * hf + 2], ga[4 * hf + 3]), xqv);
            if (cross) {   // key r against the second half's reference: its dk term and -(its dGam side)
              const float4 ycv = make_float4(yc[c], yc[c + 1], yc[c + 2], yc[c + 3]);
              const float4 g47 = g4[sw4(47, F)];
              km[2 * u + hf] = f4mul(f4exp(make_float4(g47.x - gam.x, g47.y - gam.y, g47.z - gam.z, g47.w - gam.w)), ycv);
              const float4 pc = f4mul(make_float4(gc[4 * hf], gc[4 * hf + 1], gc[4 * hf + 2], gc[4 * hf + 3]), ycv);
              qa = make_float4(qa.x - pc.x, qa.y - pc.y, qa.z - pc.z, qa.w - pc.w);
            }
            qdg4[sw4(r, F)] = qa;
            slab_put(slab, lane, 2 * u + hf, add);
          }
        }
        // onto the state part's dq, no read back
        slab_rows_out<true>(slab, dqp + base_row + (size_t)(32 * (qd - 2)) * row_stride + c0, row_stride,
                            L - 32 * (qd - 2), lane);
        if (cross) {   // the cross rows' part of dk for keys 0..31
#pragma unroll
          for (int j = 0; j < 8; ++j) slab_put(slab, lane, j, km[j]);
          slab_rows_out<true>(slab, dkp_ + base_row + c0, row_stride, L, lane);
        }
      }
    } else if (!aborted) {
      const int t = 32 * qd + lane;
      const int ref = t < 32 ? 15 : 47;
      const int gbrow = t < 32 ? t : 32 + t;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int c0 = hw * 64 + 32 * half;
        float xk[32], yo[32];
        tc::tmem_ld32(tl + 0 + c0, xk);
        tc::tmem_ld32(tl + 128 + c0, yo);
        tc::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float ga[8], gb[8];
          tile8(Lay::GA, 128, t, (c0 >> 3) + u, ga);
          tile8(Lay::GB, 96, gbrow, (c0 >> 3) + u, gb);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int F = (c0 >> 2) + 2 * u + hf, c = 8 * u + 4 * hf;
            const float4 gam = g4[sw4(t, F)], gref = g4[sw4(ref, F)];
            const float4 dlt = make_float4(gam.x - gref.x, gam.y - gref.y, gam.z - gref.z, gam.w - gref.w);
            const float4 xkv = make_float4(xk[c], xk[c + 1], xk[c + 2], xk[c + 3]);
            const float4 yov = make_float4(yo[c], yo[c + 1], yo[c + 2], yo[c + 3]);
            const float4 dkp = f4mul(f4exp(dlt), xkv);
            const float4 dkm = f4mul(f4exp(make_float4(-dlt.x, -dlt.y, -dlt.z, -dlt.w)), yov);
            const float4 pa = f4mul(make_float4(ga[4 * hf], ga[4 * hf + 1], ga[4 * hf + 2], ga[4 * hf + 3]), xkv);
            const float4 pb = f4mul(make_float4(gb[4 * hf], gb[4 * hf + 1], gb[4 * hf + 2], gb[4 * hf + 3]), yov);
            kdg4[sw4(t, F)] = make_float4(pa.x - pb.x, pa.y - pb.y, pa.z - pb.z, pa.w - pb.w);
            slab_put(slab, lane, 2 * u + hf, make_float4(dkp.x + dkm.x, dkp.y + dkm.y, dkp.z + dkm.z, dkp.w + dkm.w));
          }
        }
        slab_rows_out<true>(slab, dkp_ + base_row + (size_t)(32 * qd) * row_stride + c0, row_stride, L - 32 * qd,
                            lane);
      }
    }
    tc::fence_smem_to_async();
    __syncthreads();
    // The Gram tiles and Gam are consumed: the next item's inputs land during the scan.
    if (!aborted && has_next) {
      issue_g(h2, t02, L2, p + gridDim.x, true, kGBytes + kKqvBytes);
      if (tid == 32) issue_kqv(h2, t02);
      pre = true;
    }
    // dg += reverse cumulative sum of dGam: two threads per channel, 32 rows each.
    if (!aborted) {
      const int ch = tid & 127, hf = tid >> 7;
      const float *qdg = reinterpret_cast<const float *>(qdg4), *kdg = reinterpret_cast<const float *>(kdg4);
      float *sred = s_Y;
      float dgam[32], part = 0.f;   // dGam of rows 32 hf + i, kept for the suffix sums
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = 32 * hf + i;
        dgam[i] = qdg[sw(r, ch)] + kdg[sw(r, ch)];
        part += dgam[i];
      }
      sred[hf * 128 + ch] = part;
      __syncthreads();
      float *dgp = a.dg;
      float suffix = hf == 0 ? sred[128 + ch] : 0.f;
#pragma unroll
      for (int i = 31; i >= 0; --i) {
        const int r = 32 * hf + i;
        suffix += dgam[i];
        if (r < L) atomicAdd(dgp + base_row + (size_t)r * row_stride + ch, suffix);
      }
    }
    if (!aborted && tid < L) a.dbeta[(size_t)(t0 + tid) * H + h] = s_db[tid];
  }
  // Every reader of this item's shared memory and tensor memory is done
  // before the next item's copies land.
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  }   // items

  if (aborted) {
    report(a.dev_status, KDA_ERR_TIMEOUT);
    wait_timed(bar, phase, a.wait_ns);
    wait_timed(tbar, tphase, a.wait_ns);
    wait_timed(cbar, cphase, a.wait_ns);
    if (PART == 0 && s0pend) wait_timed(s0bar, s0phase, a.wait_ns);
    if (PART == 0 && rpend) wait_timed(rbar, rphase, a.wait_ns);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace
}  // namespace kda

namespace kda {
namespace {

// pref[n] = chunks of the sequences before n, prefck[n] = their full chunks
// (the states the forward stores every 64 tokens); one warp.
__global__ void bwd_prefix_kernel(const int32_t *__restrict__ cu, int N, int64_t *pref,
                                  int64_t *prefck) {
  const int lane = threadIdx.x;
  int64_t carry = 0, carryck = 0;
  if (lane == 0) { pref[0] = 0; prefck[0] = 0; }
  for (int base = 0; base < N; base += 32) {
    const int i = base + lane;
    const int64_t len = i < N ? (int64_t)cu[i + 1] - cu[i] : 0;
    int64_t v = (len + kC - 1) / kC, w = len / kC;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t tv = __shfl_up_sync(0xffffffffu, v, o), tw = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) { v += tv; w += tw; }
    }
    if (i < N) { pref[i + 1] = carry + v; prefck[i + 1] = carryck + w; }
    carry += __shfl_sync(0xffffffffu, v, 31);
    carryck += __shfl_sync(0xffffffffu, w, 31);
  }
}

// The initial states as BF16 operand tiles, in the layout of the forward's
// checkpoint tiles (128-byte swizzled [key channel][value column]).
__global__ void __launch_bounds__(kThreads)
bwd_init_tiles_kernel(const float *__restrict__ init, uint8_t *__restrict__ tiles) {
  const int unit = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float *src = init + (size_t)unit * kD * kD;
  uint8_t *dst = tiles + (size_t)unit * 32768;
  constexpr int kRows = kD / (kThreads / 32);   // rows per warp: all loads first, then the stores
  float4 x[kRows];
#pragma unroll
  for (int i = 0; i < kRows; ++i)
    x[i] = reinterpret_cast<const float4 *>(src + (size_t)(warp + 8 * i) * kD)[lane];
#pragma unroll
  for (int i = 0; i < kRows; ++i)
    *reinterpret_cast<uint2 *>(dst + tc::tile_offset(128, warp + 8 * i, lane >> 1) + 8 * (lane & 1)) =
        make_uint2(tc::pack_bf16(x[i].x, x[i].y), tc::pack_bf16(x[i].z, x[i].w));
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BwdWs {
  size_t pk, ck, s0i, tt, dsl, ndu, dot, dtp, oscr, pref, prefck, items, total;
};

BwdWs bwd_ws_layout(int N, int H, int64_t T) {
  const size_t P = (size_t)H * (size_t)((T + (int64_t)(kC - 1) * N) / kC);   // packets, upper bound
  BwdWs w;
  size_t off = 0;
  w.pk = off;     off += align256(P * Pk::BYTES + 256);
  w.ck = off;     off += align256((size_t)(T / kC) * H * 32768);      // BF16 state tiles
  w.s0i = off;    off += align256((size_t)N * H * 32768);             // initial states, same layout
  w.tt = off;     off += align256(P * 16384);                         // T, (I + M)^-1 per packet
  w.dsl = off;    off += align256(P * 32768);
  w.ndu = off;    off += align256(P * 16384);
  w.dot = off;    off += align256(P * 16384);
  w.dtp = off;    off += align256(P * kDtpBytes);
  w.oscr = off;   off += align256((size_t)T * H * kD * 2);
  w.pref = off;   off += align256((size_t)(N + 1) * 8);
  w.prefck = off; off += align256((size_t)(N + 1) * 8);
  w.items = off;  off += align256(P * sizeof(ItemRec));
  w.total = off + 256;
  return w;
}

}  // namespace

bool backward_tc_supported(int dtype, int dk, int dv, int N) {
  return dtype == KDA_DTYPE_BF16 && dk == kD && dv == kD && prefill_split_supported(N);
}

size_t backward_tc_workspace_bytes(int N, int H, int64_t T) { return bwd_ws_layout(N, H, T).total; }

cudaError_t launch_backward_tc(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *init, const int32_t *cu,
                               const float *dout, const float *dfin, float *dq, float *dk,
                               float *dv, float *dg, float *dbeta, float *dinit, void *workspace,
                               int N, int H, int64_t T, int32_t *dev_status, cudaStream_t stream,
                               int num_sms) {
  if (split_packet_bytes() != Pk::BYTES) return cudaErrorInvalidValue;
  const BwdWs w = bwd_ws_layout(N, H, T);
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~(uintptr_t)255);
  uint8_t *pk = base + w.pk;
  uint8_t *ck = base + w.ck;
  uint8_t *s0i = base + w.s0i;
  uint8_t *tt = base + w.tt;
  uint8_t *dsl = base + w.dsl;
  uint8_t *ndu = base + w.ndu;
  uint8_t *dot = base + w.dot;
  uint8_t *dtp = base + w.dtp;
  void *oscr = base + w.oscr;
  int64_t *pref = reinterpret_cast<int64_t *>(base + w.pref);
  int64_t *prefck = reinterpret_cast<int64_t *>(base + w.prefck);
  ItemRec *items = reinterpret_cast<ItemRec *>(base + w.items);
  const uint64_t wait_ns = 2000000000ull;

  // Forward recomputation: the two-pass prefill in one window keeps every
  // intra-chunk packet in the workspace and stores the state every 64 tokens.
  cudaError_t e = launch_prefill_split_ex(q, k, v, g, beta, init, cu, oscr, nullptr, kC, nullptr,
                                          ck, tt, N, H, T, pk, w.ck - w.pk, dev_status, stream, num_sms);
  if (e != cudaSuccess) return e;
  if (init) {
    bwd_init_tiles_kernel<<<(unsigned)((int64_t)N * H), kThreads, 0, stream>>>(init, s0i);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  bwd_prefix_kernel<<<1, 32, 0, stream>>>(cu, N, pref, prefck);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const int64_t P_max = (int64_t)H * ((T + (int64_t)(kC - 1) * N) / kC);
  bwd_dout_tiles_kernel<<<(unsigned)((P_max + 1) / 2), kThreads, 0, stream>>>(dout, cu, pref, N, H, dot, items);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  TmaMaps maps;
  if (!make_input_maps(&maps, q, k, v, g, H, T) ||
      !make_map(&maps.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, H, T, 64, 64,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&maps.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, H, T, 64, 64,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  const size_t smem_c = BChainLayout::TOTAL + 1024;
  e = cudaFuncSetAttribute(bwd_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_c);
  if (e != cudaSuccess) return e;
  bwd_chain_kernel<<<(unsigned)((int64_t)N * H), kThreads, smem_c, stream>>>(
      pk, dot, cu, dfin, dinit, dsl, ndu, N, H, dev_status, wait_ns);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  BwdItemArgs a;
  a.beta = beta; a.s0_init = init ? s0i : nullptr; a.s0_ck = ck; a.cu = cu; a.pref = pref; a.prefck = prefck;
  a.dsl = dsl; a.ndu = ndu; a.dot = dot; a.dtp = dtp; a.tt = tt; a.items = items;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta;
  a.N = N; a.H = H; a.dev_status = dev_status; a.wait_ns = wait_ns;
  const size_t smem_i = BItemLayout::TOTAL + 1024;
  e = cudaFuncSetAttribute(bwd_item_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_i);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_item_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_i);
  if (e != cudaSuccess) return e;
  bwd_item_kernel<0><<<num_sms, kThreads, smem_i, stream>>>(maps, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_item_kernel<1><<<num_sms, kThreads, smem_i, stream>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace kda
