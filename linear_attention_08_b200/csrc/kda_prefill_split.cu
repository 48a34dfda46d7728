// KDA chunked prefill in two passes on the 5th-generation tensor cores (sm_100a).
//
// The chunked form ("LLM - Semianalysis, Kimi K3 아키텍처", Methods 1, FlashKDA;
// "MoonshotAI/Kimi-K3 딥다이브", section 4-1) splits every chunk's work into a
// part that depends only on the chunk's own inputs and a short part that
// needs the state entering the chunk.  With Gam_r = sum_{s<=r} g_s and
// T = (I + M)^-1 diag(beta) as in the fused kernel:
//
//   W = T Ktilde,  U = T V                              (state-free)
//   V_new = U - W S0                                    (per chunk, serial)
//   O     = Qtilde S0 + P V_new
//   S     = Diag(exp(Gam_last)) S0 + Khat^T V_new
//
// (W S0 = T Ktilde S0, so V_new = T (V - Ktilde S0) is the fused kernel's U.)
//
// Pass 1 (intra_kernel) runs every (chunk, head) pair independently: gates,
// the gated Gram products, the UT transform and the products T Ktilde and
// T V; it writes one "packet" per pair to a workspace in global memory, its
// MMA operands already in the 128-byte-swizzled shared-memory tile layout.
// Two CTAs share an SM, so one's tensor-core and load waits overlap the
// other's SIMT work.
//
// Pass 2 (chain_kernel) walks each (sequence, head, value slice) chunk by
// chunk.  Per chunk it bulk-copies the packet (double or triple buffered) and
// runs two tensor-core steps and two epilogues:
//   [W; Qtilde] S0 -> acc1         V_new = U - (acc1 rows 0..63)
//   acc1 += [*; P] V_new,  acc2 = Khat^T V_new,  S = d * S + acc2 (FP32, TMEM)
// The FP32 state lives in tensor memory; its BF16 copy is the MMA operand.
//
// Long inputs are processed in windows of chunks so that the workspace stays
// within the size the caller grants; the state is carried between windows in
// FP32 through global memory.
#include <cuda.h>

#include "kda_common.cuh"
#include "kda_tc_util.cuh"
#include "kda_tma.cuh"

namespace kda {
namespace {

constexpr int kC = 64;
constexpr int kDK = 128;
constexpr int kDV = 128;
constexpr int kThreads = 256;
constexpr int kLd = 68;
constexpr int kMaxSeqs = 1024;   // sequences per call on this path

// One packet: what the chain needs from one (chunk, head).
struct Packet {
  static constexpr uint32_t WQ = 0;        // [128][128] bf16 tile: W rows 0..63, Qtilde rows 64..127
  static constexpr uint32_t KH = 32768;    // [64][128] bf16 tile: Khat (tokens x key channels)
  static constexpr uint32_t U = 49152;     // [64][128] bf16 tile: U = T V (tokens x value columns)
  static constexpr uint32_t P = 65536;     // [64][64] bf16 tile: P (lower triangle, diagonal included)
  static constexpr uint32_t D = 73728;     // float[128]: exp(Gam) at the chunk's last token
  static constexpr uint32_t BYTES = 74240;
};

// ---------------------------------------------------------------------------
// Pass 1: intra-chunk products
// ---------------------------------------------------------------------------
struct IntraLayout {
  // 64 KB region used in turn for: the raw inputs (k and q land by TMA in the
  // rows of the Gram A tile that their scaled versions replace; g, fp32, in
  // the upper half); the Gram operands and the gate factors; the solve
  // scratch and the V tile.
  static constexpr uint32_t STG_G = 0;       // float [64][128] g
  static constexpr uint32_t GA = 32768;      // [128][128] Gram A, K-major: k rows 0..63, q rows 64..127
  static constexpr uint32_t GB = 0;          // [96][128]  Gram B, K-major (over the consumed g)
  static constexpr uint32_t CST = 24576;     // float [2][6][128] gate factors
  static constexpr uint32_t MM = 0;          // float [64][68] M
  static constexpr uint32_t XM = 17408;      // float [64][68] (I + M)^-1
  static constexpr uint32_t YS = 34816;      // float [2][16][17]
  static constexpr uint32_t ZS = 36992;      // float [32][36]
  static constexpr uint32_t MT = 41600;      // float [32][33] M_(1,0)^T
  static constexpr uint32_t VT = 49152;      // [64][128] V tile (MN-major B), loaded after the Gram MMA
  static constexpr uint32_t KT = 65536;      // [64][128] Ktilde tile (MN-major B)
  static constexpr uint32_t TP = 81920;      // [128][64] T (rows 0..63) as K-major A
  static constexpr uint32_t RED = TP;        // float [8][128] scan partials (before T exists)
  static constexpr uint32_t BETA = 98304;    // float [64]
  static constexpr uint32_t PREF = BETA + 256;                    // int [kMaxSeqs + 1]
  static constexpr uint32_t CUS = PREF + 4 * (kMaxSeqs + 1);      // int [kMaxSeqs + 1] cu_seqlens
  static constexpr uint32_t BAR = (CUS + 4 * (kMaxSeqs + 1) + 7) & ~7u;    // MMA completion
  static constexpr uint32_t TBAR = BAR + 8;                       // q, k landed
  static constexpr uint32_t VBAR = BAR + 16;                      // v landed
  static constexpr uint32_t GBAR = BAR + 24;                      // g landed
  static constexpr uint32_t TMEM_SLOT = BAR + 32;
  static constexpr uint32_t NEXT = BAR + 40;                      // int64 [2][2]: the next item's t0, (L, h)
  static constexpr uint32_t TOTAL = NEXT + 32;
  static_assert(MT + 32 * 33 * 4 <= VT, "solve scratch overlaps the V tile");
  static_assert(VT >= GA && VT + 16384 <= GA + 32768, "the V tile must lie in the consumed Gram A tile");
  static_assert(MT + 32 * 33 * 4 <= 65536 && STG_G + 32768 <= GA, "g staging and the solve scratch");
  static_assert(CST + 6144 <= GA, "gate factors overflow into the Gram A tile");
  static_assert(GB + 96 * 256 <= CST, "Gram B overlaps the gate factors");
};

// 16-byte store of 8 floats as bf16 into shared memory, as a plain C++ store
// (the compiler may schedule loads around it; the proxy fences that publish
// the tiles to the tensor core are ordered after it).
__device__ __forceinline__ void st_chunk_s(uint8_t *dst, const float *x) {
  *reinterpret_cast<uint4 *>(dst) = make_uint4(tc::pack_bf16(x[0], x[1]), tc::pack_bf16(x[2], x[3]),
                                               tc::pack_bf16(x[4], x[5]), tc::pack_bf16(x[6], x[7]));
}

// Chunks of sequence n that fall in the window [jw0, jw0 + wc).
__device__ __forceinline__ int64_t window_chunks(const int32_t *cu, int n, int64_t jw0, int64_t wc) {
  const int64_t nch = ((int64_t)cu[n + 1] - cu[n] + kC - 1) / kC;
  const int64_t c = nch - jw0;
  return c <= 0 ? 0 : (c < wc ? c : wc);
}

// g (fp32, staging rows of 512 bytes) and beta (4-byte async copies, zero
// past L): needed first by the next chunk, and their space is free once T is
// formed.
__device__ __forceinline__ void intra_issue_g(uint32_t sb, const TmaMaps &maps, const float *beta,
                                              int64_t t0, int L, int H, int h, int tid) {
  using Lay = IntraLayout;
  if (tid == 32) {
    const uint32_t bar = sb + Lay::GBAR;
    mbar_expect_tx(bar, 64 * 512);
    tma_load_3d(sb + Lay::STG_G, &maps.g, 0, h, (int)t0, bar);
  }
  if (tid >= 64 && tid < 64 + kC) {
    const int r = tid - 64;
    const bool ok = r < L;
    cp_async4(sb + Lay::BETA + 4 * r, beta + (ok ? (size_t)(t0 + r) * H + h : 0), ok);
  }
  cp_async_commit();
}

// q and k come through maps with the v layout (box 64 x 64, 128-byte swizzle):
// each box is one 64-row column block, i.e. rows 0..63 (k) or 64..127 (q) of a
// column block of the Gram A tile, whose space holds the V tile until the last
// product of the previous chunk is done.
__device__ __forceinline__ void intra_issue_qk(uint32_t sb, const TmaMaps &maps, int64_t t0,
                                               int h, int tid) {
  using Lay = IntraLayout;
  if (tid == 32) {
    const uint32_t bar = sb + Lay::TBAR;
    mbar_expect_tx(bar, 64 * 512);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      tma_load_3d(sb + Lay::GA + b * 16384, &maps.k, 64 * b, h, (int)t0, bar);
      tma_load_3d(sb + Lay::GA + b * 16384 + 8192, &maps.q, 64 * b, h, (int)t0, bar);
    }
  }
}

// Work item p of the window -> (sequence, head, chunk); see the packet order
// in launch_prefill_split.
struct Item {
  int n, h, L;
  int64_t j, t0;
};

__device__ __forceinline__ Item decode_item(int p, const int32_t *s_pref, const int32_t *cu, int N,
                                            int H, int64_t jw0) {
  int lo = 0, hi = N - 1;
  while (lo < hi) {   // last sequence whose first packet is at or before p
    const int mid = (lo + hi + 1) >> 1;
    if (s_pref[mid] <= p) lo = mid; else hi = mid - 1;
  }
  Item it;
  it.n = lo;
  const int cnt = (s_pref[lo + 1] - s_pref[lo]) / H;
  const int r = p - s_pref[lo];
  it.h = r / cnt;
  it.j = jw0 + (r - it.h * cnt);
  const int64_t T_n = (int64_t)cu[lo + 1] - cu[lo];
  it.t0 = cu[lo] + kC * it.j;
  const int64_t rem = T_n - kC * it.j;
  it.L = (int)(rem < kC ? rem : kC);
  return it;
}

__global__ void __launch_bounds__(kThreads, 2)
intra_kernel(const __grid_constant__ TmaMaps maps, const float *__restrict__ beta,
             const int32_t *__restrict__ cu, int N, int H, int64_t jw0, int64_t wc,
             uint8_t *__restrict__ ws, uint8_t *__restrict__ tt_out, int32_t *dev_status,
             uint64_t wait_ns) {
  using Lay = IntraLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t *sp = smem_raw + (sb - sraw);
  float *s_beta = reinterpret_cast<float *>(sp + Lay::BETA);
  float *s_red = reinterpret_cast<float *>(sp + Lay::RED);
  float *s_cst = reinterpret_cast<float *>(sp + Lay::CST);
  float *s_M = reinterpret_cast<float *>(sp + Lay::MM);
  float *s_X = reinterpret_cast<float *>(sp + Lay::XM);
  float *s_Y = reinterpret_cast<float *>(sp + Lay::YS);
  float *s_Z = reinterpret_cast<float *>(sp + Lay::ZS);
  float *s_MT = reinterpret_cast<float *>(sp + Lay::MT);
  int32_t *s_pref = reinterpret_cast<int32_t *>(sp + Lay::PREF);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sp + Lay::BAR);
  uint64_t *tbar = reinterpret_cast<uint64_t *>(sp + Lay::TBAR);
  uint64_t *vbar = reinterpret_cast<uint64_t *>(sp + Lay::VBAR);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hw = warp >> 2;

  int32_t *s_cu = reinterpret_cast<int32_t *>(sp + Lay::CUS);
  for (int n = tid; n <= N; n += kThreads) s_cu[n] = cu[n];
  // Packets of the window, sequence by sequence: s_pref[n] = first packet of n.
  for (int n = tid; n < N; n += kThreads) s_pref[n + 1] = (int32_t)(window_chunks(cu, n, jw0, wc) * H);
  if (tid == 0) s_pref[0] = 0;
  __syncthreads();
  if (warp == 0) {
    int32_t carry = 0;
    for (int base = 1; base <= N; base += 32) {
      const int i = base + lane;
      int32_t v = i <= N ? s_pref[i] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      if (i <= N) s_pref[i] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
  const int total = s_pref[N];
  if ((int)blockIdx.x >= total) return;

  uint64_t *gbar = reinterpret_cast<uint64_t *>(sp + Lay::GBAR);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(tbar, 1);
    mbar_init(vbar, 1);
    mbar_init(gbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.q)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.g)) : "memory");
  }
  if (warp == 0) tc::tmem_alloc(sb + Lay::TMEM_SLOT, 256);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + Lay::TMEM_SLOT);
  const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);

  uint32_t phase = 0, tphase = 0, vphase = 0, gphase = 0;
  bool aborted = false;
  int p = blockIdx.x;
  // The next item's place is found by one thread while the Gram product runs
  // (its search and divisions are off every other thread's path) and handed
  // over through shared memory, in two slots used in turn.
  int64_t *s_next = reinterpret_cast<int64_t *>(sp + Lay::NEXT);
  int slot = 0;
  int64_t cur_t0;
  int cur_L, cur_h;
  {
    const Item it = decode_item(p, s_pref, s_cu, N, H, jw0);
    intra_issue_g(sb, maps, beta, it.t0, it.L, H, it.h, tid);
    intra_issue_qk(sb, maps, it.t0, it.h, tid);
    cur_t0 = it.t0;
    cur_L = it.L;
    cur_h = it.h;
  }

  for (; p < total; p += gridDim.x) {
    const bool more = p + (int)gridDim.x < total;
    const int L = cur_L, h = cur_h;
    const int64_t t0 = cur_t0;
    uint8_t *pk = ws + (size_t)p * Packet::BYTES;

    cp_async_wait_all();
    if (tid == 0) bulk_wait_read();   // the previous item's W and U have left KT and TP
    if (__syncthreads_or(!wait_timed(gbar, gphase, wait_ns))) { aborted = true; break; }
    gphase ^= 1;

    // ---------------- gate prep ----------------
    // Warp w owns rows 8w..8w+7 (half hf = w / 4), lane l owns channels 4l..4l+3
    // (two pairs, handled by the paired FP32 instructions, each lane of which
    // rounds like the scalar one): per row one 8-byte piece of each 16-byte tile
    // chunk; the gate factors of the lane's channels stay in registers.
    {
      const int hf = warp >> 2, cq = lane >> 1, sub = (lane & 1) * 8;
      float2 gm[8][2];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * warp + i;
        const float4 a = r < L ? *reinterpret_cast<const float4 *>(sp + Lay::STG_G + r * 512 + lane * 16)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        gm[i][0] = make_float2(a.x, a.y);
        gm[i][1] = make_float2(a.z, a.w);
      }
#pragma unroll
      for (int i = 1; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) gm[i][j] = __fadd2_rn(gm[i][j], gm[i - 1][j]);
      *reinterpret_cast<float4 *>(s_red + warp * 128 + 4 * lane) =
          make_float4(gm[7][0].x, gm[7][0].y, gm[7][1].x, gm[7][1].y);
      __syncthreads();
      // One lane per channel: exclusive scan of the 8 row-group totals, the cumulative
      // decay at rows 15, 31, 47, 63, and the channel's gate factors for both halves.
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
        // Row r of half hf is scaled against ref = Gam_15 (hf 0) or Gam_47 (hf 1);
        // the products are grouped exactly as in the fused kernel (no intermediate
        // underflows unless the exact value is itself far below the BF16 rounding).
        // Slots: -ref, fk, fk2, fh, fh2, cb; fk = 1 in the first half and fh2 = 1 in
        // the second, so (x fk) fk2 and (y fh) fh2 serve both halves exactly.
        float f[12];
        f[0] = -G15; f[1] = 1.f; f[2] = __expf(G15);
        f[3] = __expf(G31 - G15); f[4] = __expf(G63 - G31); f[5] = __expf(G47 - G15);
        f[6] = -G47; f[7] = __expf(G47 - G31); f[8] = __expf(G31);
        f[9] = __expf(G63 - G47); f[10] = 1.f; f[11] = 0.f;
#pragma unroll
        for (int j = 0; j < 12; ++j) s_cst[j * 128 + ch] = f[j];
        reinterpret_cast<float *>(pk + Packet::D)[ch] = __expf(G63);
      }
      // q and k must have landed too before the rows are scaled.
      if (__syncthreads_or(!wait_timed(tbar, tphase, wait_ns))) { aborted = true; break; }
      tphase ^= 1;
      float2 nref[2], fk[2], fk2[2];   // fh, fh2, cb (used once per row) stay in shared memory
      {
        auto ld4 = [&](int j, float2 *d) {
          const float4 v = *reinterpret_cast<const float4 *>(s_cst + (hf * 6 + j) * 128 + 4 * lane);
          d[0] = make_float2(v.x, v.y);
          d[1] = make_float2(v.z, v.w);
        };
        float2 base[2];
        const float4 bv = *reinterpret_cast<const float4 *>(s_red + warp * 128 + 4 * lane);
        base[0] = make_float2(bv.x, bv.y);
        base[1] = make_float2(bv.z, bv.w);
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 2; ++j) gm[i][j] = __fadd2_rn(gm[i][j], base[j]);
        ld4(0, nref); ld4(1, fk); ld4(2, fk2);
      }
      auto st4 = [&](uint8_t *dst, const float2 *x) {
        *reinterpret_cast<uint2 *>(dst) = make_uint2(tc::pack_bf16(x[0].x, x[0].y), tc::pack_bf16(x[1].x, x[1].y));
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
        {   // raw k and q of this row, replaced below by k x and q x
          const bool in = r < L;
          const uint2 z2 = make_uint2(0, 0);
          const uint2 kv = in ? *reinterpret_cast<const uint2 *>(sp + Lay::GA + tc::tile_offset(128, r, cq) + sub) : z2;
          const uint2 qv = in ? *reinterpret_cast<const uint2 *>(sp + Lay::GA + tc::tile_offset(128, 64 + r, cq) + sub) : z2;
          un4(kv, kk);
          un4(qv, qq);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float2 d = __fadd2_rn(gm[i][j], nref[j]);
          x[j] = make_float2(__expf(d.x), __expf(d.y));   // exp(Gam_r - ref), within [e^-80, e^80]
          y[j] = make_float2(rcp(x[j].x), rcp(x[j].y));   // exp(ref - Gam_r)
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(kk[j], x[j]);
        st4(sp + Lay::GA + tc::tile_offset(128, r, cq) + sub, t);
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(qq[j], x[j]);
        st4(sp + Lay::GA + tc::tile_offset(128, 64 + r, cq) + sub, t);
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(kk[j], y[j]);
        st4(sp + Lay::GB + tc::tile_offset(96, hf ? 32 + r : r, cq) + sub, t);
        if (!hf) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float2 cb = reinterpret_cast<const float2 *>(s_cst + (hf * 6 + 5) * 128 + 4 * lane)[j];
            t[j] = __fmul2_rn(kk[j], __fmul2_rn(y[j], cb));
          }
          st4(sp + Lay::GB + tc::tile_offset(96, 32 + r, cq) + sub, t);
        }
        // Ktilde, Qtilde: exp(Gam_r) = (x fk) fk2.
#pragma unroll
        for (int j = 0; j < 2; ++j) x[j] = __fmul2_rn(__fmul2_rn(x[j], fk[j]), fk2[j]);
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(kk[j], x[j]);
        st4(sp + Lay::KT + tc::tile_offset(64, r, cq) + sub, t);
#pragma unroll
        for (int j = 0; j < 2; ++j) t[j] = __fmul2_rn(qq[j], x[j]);
        st4(pk + Packet::WQ + tc::tile_offset(128, 64 + r, cq) + sub, t);
        // Khat: exp(Gam_last - Gam_r) = (y fh) fh2.
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float2 fh = reinterpret_cast<const float2 *>(s_cst + (hf * 6 + 3) * 128 + 4 * lane)[j];
          const float2 fh2 = reinterpret_cast<const float2 *>(s_cst + (hf * 6 + 4) * 128 + 4 * lane)[j];
          t[j] = __fmul2_rn(kk[j], __fmul2_rn(__fmul2_rn(y[j], fh), fh2));
        }
        st4(pk + Packet::KH + tc::tile_offset(64, r, cq) + sub, t);
      }
      tc::fence_smem_to_async();
      __syncthreads();
    }

    // ---------------- gated Gram products: one [128 x 96 x 128] MMA ----------------
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 96, 0, 0);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem, tc::desc_kmajor(sb + Lay::GA, 128, s2), tc::desc_kmajor(sb + Lay::GB, 96, s2),
                     id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (tid == 224 && more) {
      const Item nx = decode_item(p + (int)gridDim.x, s_pref, s_cu, N, H, jw0);
      s_next[2 * (slot ^ 1)] = nx.t0;
      s_next[2 * (slot ^ 1) + 1] = ((int64_t)nx.h << 32) | (uint32_t)nx.L;
    }
    if (__syncthreads_or(!wait_timed(bar, phase, wait_ns))) { aborted = true; break; }
    phase ^= 1;
    tc::fence_after_sync();
    // The Gram operands are consumed: load this chunk's V tile into their place.
    if (tid == 32) {
      const uint32_t vb = sb + Lay::VBAR;
      mbar_expect_tx(vb, 64 * 256);
      tma_load_3d(sb + Lay::VT, &maps.v, 0, h, (int)t0, vb);
      tma_load_3d(sb + Lay::VT + 8192, &maps.v, 64, h, (int)t0, vb);
    }

    // Gram rows: lane m = row m.  k rows -> FP32 M (scaled by beta_r, strictly
    // lower); q rows -> P (lower with diagonal), straight to the packet.
    {
      const int m = 32 * qd + lane, part = m >> 6, r = m & 63, second = r >> 5;
      const int i0 = second ? 32 * hw : (hw ? 32 : 0);
      float a[32];
      if (second || hw == 0) {
        tc::tmem_ld32(tl + (second ? 32 + 32 * hw : 0), a);
        tc::tmem_wait_ld();
      }
      const bool zero = !second && hw;
      if (part == 0) {   // 16-byte stores: rows are 272 bytes apart, so 8 lanes hit 8 distinct slots
        const float br = s_beta[r];
        float4 *dst = reinterpret_cast<float4 *>(s_M + r * kLd + i0);
        auto mv = [&](int j) { return (!zero && i0 + j < r) ? br * a[j] : 0.f; };
#pragma unroll
        for (int j = 0; j < 32; j += 4) dst[j >> 2] = make_float4(mv(j), mv(j + 1), mv(j + 2), mv(j + 3));
        if (second && i0 == 0)
#pragma unroll
          for (int j = 0; j < 32; ++j) s_MT[j * 33 + (r - 32)] = br * a[j];
      } else {   // P rows go to rows 64..127 of the TP tile, then to the packet in one bulk copy
#pragma unroll
        for (int j = 0; j < 32; ++j) a[j] = (!zero && i0 + j <= r) ? a[j] : 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_chunk_s(sp + Lay::TP + tc::tile_offset(128, 64 + r, (i0 >> 3) + cc), a + 8 * cc);
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      bulk_store(pk + Packet::P, sb + Lay::TP + 8192, 8192);
      bulk_commit();
    }

    // ---------------- UT transform: (I + M)^-1 on 16x16 diagonal blocks ----------------
    if (qd >= 2) {
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
        for (int i = 0; i < 8; ++i) m[i] = mrow[i * kLd + sidx];
        const float xs = __shfl_sync(0xffffffffu, x[sidx & 7], c + 16 * (sidx >> 3));
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = fmaf(-m[i], xs, x[i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) s_X[(o + 8 * hf + i) * kLd + o + c] = x[i];
      if ((blk & 1) == 0)
#pragma unroll
        for (int i = 0; i < 8; ++i) s_X[(o + 8 * hf + i) * kLd + o + 16 + c] = 0.f;
    }
    __syncthreads();
    // Level 1: the 32x32 inverse of each half.
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
    // Level 2: X_(1,0) = -H1 M_(1,0) H0 with triangular trip counts.
    {
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
      const int r2 = 4 * warp + (lane >> 3), c2 = 4 * (lane & 7);
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s2 = 0; s2 < 4 * warp + 4; ++s2) {
        const float a = s_X[(32 + r2) * kLd + 32 + s2];
        const float4 zv = *reinterpret_cast<const float4 *>(s_Z + s2 * 36 + c2);
        w.x = fmaf(a, zv.x, w.x); w.y = fmaf(a, zv.y, w.y);
        w.z = fmaf(a, zv.z, w.z); w.w = fmaf(a, zv.w, w.w);
      }
      *reinterpret_cast<float4 *>(s_X + (32 + r2) * kLd + c2) = make_float4(-w.x, -w.y, -w.z, -w.w);
      if (tid == 0) bulk_wait_read();   // the P copy has left rows 64..127 of TP
      __syncthreads();
    }
    // T_ri = X_ri beta_i (i <= r), in rows 0..63 and again in rows 64..127 of the
    // K-major A tile, so that the product rows reach all four TMEM lane quadrants.
    // With `tt_out` (the backward's forward recomputation) T and (I + M)^-1
    // also go to global memory as [64][64] BF16 tiles, 16 KB per item.
    for (int e = tid; e < 64 * 8; e += kThreads) {
      const int row = e >> 3, ch = e & 7;
      float val[8], xv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = 8 * ch + u;
        xv[u] = i <= row ? s_X[row * kLd + i] : 0.f;
        val[u] = xv[u] * s_beta[i];
      }
      st_chunk_s(sp + Lay::TP + tc::tile_offset(128, row, ch), val);
      st_chunk_s(sp + Lay::TP + tc::tile_offset(128, 64 + row, ch), val);
      if (tt_out) {
        uint8_t *tt = tt_out + (size_t)p * 16384 + tc::tile_offset(64, row, ch);
        *reinterpret_cast<uint4 *>(tt) = make_uint4(tc::pack_bf16(val[0], val[1]), tc::pack_bf16(val[2], val[3]),
                                                    tc::pack_bf16(val[4], val[5]), tc::pack_bf16(val[6], val[7]));
        *reinterpret_cast<uint4 *>(tt + 8192) = make_uint4(tc::pack_bf16(xv[0], xv[1]), tc::pack_bf16(xv[2], xv[3]),
                                                           tc::pack_bf16(xv[4], xv[5]), tc::pack_bf16(xv[6], xv[7]));
      }
    }
    tc::fence_smem_to_async();
    if (__syncthreads_or(!wait_timed(vbar, vphase, wait_ns))) { aborted = true; break; }
    vphase ^= 1;
    // The solve scratch and beta are consumed: the next item's g and beta may land.
    const int64_t nx_t0 = s_next[2 * (slot ^ 1)], nx_lh = s_next[2 * (slot ^ 1) + 1];
    const int nx_L = (int)(uint32_t)nx_lh, nx_h = (int)(nx_lh >> 32);
    if (more) intra_issue_g(sb, maps, beta, nx_t0, nx_L, H, nx_h, tid);

    // ---------------- W = T Ktilde (columns 0..127), U = T V (128..255) ----------------
    // Rows 64..127 of the A tile repeat T: TMEM lanes 64..127 get a copy of the product.
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem, tc::desc_kmajor(sb + Lay::TP, 128, s2),
                     tc::desc_mnmajor(sb + Lay::KT, 64, s2), id, s2 > 0);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + 128, tc::desc_kmajor(sb + Lay::TP, 128, s2),
                     tc::desc_mnmajor(sb + Lay::VT, 64, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (__syncthreads_or(!wait_timed(bar, phase, wait_ns))) { aborted = true; break; }
    phase ^= 1;
    tc::fence_after_sync();
    // The V tile is consumed: the next item's q and k may land in the Gram A tile.
    if (more) intra_issue_qk(sb, maps, nx_t0, nx_h, tid);
    {   // Each warp takes one 64-column quarter of [W | U] (W -> KT tile, U -> TP tile)
        // for 32 tokens: quadrants 0, 1 read lanes 0..63, quadrants 2, 3 the copy.
      const int r = 32 * (qd & 1) + lane, quarter = 2 * (qd >> 1) + hw;
      const uint32_t dst = sb + (quarter >= 2 ? Lay::TP : Lay::KT) + (quarter & 1) * 8192;
      float a[64];
      tc::tmem_ld32(tl + 64 * quarter, *reinterpret_cast<float(*)[32]>(a));
      tc::tmem_ld32(tl + 64 * quarter + 32, *reinterpret_cast<float(*)[32]>(a + 32));
      tc::tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) st_chunk_s(sp + (dst - sb) + tc::tile_offset(64, r, cc), a + 8 * cc);
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {   // W: rows 0..63 of both column blocks of the [W; Qtilde] tile; U: whole tile
      bulk_store(pk + Packet::WQ, sb + Lay::KT, 8192);
      bulk_store(pk + Packet::WQ + 16384, sb + Lay::KT + 8192, 8192);
      bulk_store(pk + Packet::U, sb + Lay::TP, 16384);
      bulk_commit();
    }
    cur_t0 = nx_t0;
    cur_L = nx_L;
    cur_h = nx_h;
    slot ^= 1;
  }
  if (tid == 0) bulk_wait_all();

  cp_async_wait_all();
  if (aborted) {
    report(dev_status, KDA_ERR_TIMEOUT);
    wait_timed(bar, phase, wait_ns);
    wait_timed(tbar, tphase, wait_ns);
    wait_timed(vbar, vphase, wait_ns);
    wait_timed(gbar, gphase, wait_ns);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// Pass 2: the inter-chunk chain
// ---------------------------------------------------------------------------
// DVS = 128, 64 or 32 value columns per CTA.  The MN-major operand tiles of
// a 32-column slice keep the 64-column (128-byte) rows of the swizzle atom,
// half of each row used.
template <int DVS>
struct ChainLayout {
  static constexpr int NST = 2;                                   // packet buffers
  static constexpr int TW = DVS < 64 ? 64 : DVS;                  // tile width in columns
  static constexpr uint32_t S_T = 0;                              // [128][DVS] bf16 state, MN-major B
  static constexpr uint32_t VN = S_T + 128 * TW * 2;              // [64][DVS] bf16 V_new, MN-major B
  static constexpr uint32_t OBUF = VN + 64 * TW * 2;              // [64][DVS] bf16 O, rows of DVS*2 bytes
  static constexpr uint32_t STAGE0 = OBUF + 64 * TW * 2;
  // inside a stage
  static constexpr uint32_t WQ = 0;                               // [128][128] [W; Qtilde], K-major A
  static constexpr uint32_t KH = 32768;                           // [64][128] Khat, MN-major A
  static constexpr uint32_t U = 49152;                            // [64][TW] U column block (the slice's columns)
  static constexpr uint32_t UB = 64 * TW * 2;                     // its bytes
  static constexpr uint32_t P = U + UB;                           // [64][64] P = rows 64..127 of the A tile at P - 8192
  static constexpr uint32_t D = P + 8192;                         // float[128]
  static constexpr uint32_t STAGE = (D + 512 + 1023) & ~1023u;
  static constexpr uint32_t BAR = STAGE0 + NST * STAGE;           // first product done
  static constexpr uint32_t SBAR = BAR + 8;                       // state increment done
  static constexpr uint32_t OBAR = BAR + 16;                      // O accumulation done
  static constexpr uint32_t FULL = BAR + 24;                      // [NST] packet landed
  static constexpr uint32_t SCAL = FULL + 8 * NST;                // int64 [2]: first packet, checkpoint slot
  static constexpr uint32_t TMEM_SLOT = SCAL + 16;
  static constexpr uint32_t TOTAL = TMEM_SLOT + 8;
  static constexpr uint32_t TMEM_COLS = DVS == 128 ? 512 : (DVS == 64 ? 256 : 128);
  // TMEM columns: acc1 in two buffers (chunk parity), acc2, the FP32 state
  static constexpr uint32_t ACC1 = 0, ACC2 = DVS, SCOL = 2 * DVS, ACC1B = 3 * DVS;
  static constexpr uint32_t TX_BYTES = 49152 + UB + 8704;
};

template <int DVS>
__global__ void __launch_bounds__(kThreads, 1)
chain_kernel(const uint8_t *__restrict__ ws, const float *init, const int32_t *__restrict__ cu,
             __nv_bfloat16 *__restrict__ out, float *carry, int64_t interval, float *__restrict__ ck,
             uint8_t *__restrict__ ck_tiles, int N, int H, int64_t jw0, int64_t wc, int first_window,
             int32_t *dev_status, uint64_t wait_ns) {
  using Lay = ChainLayout<DVS>;
  constexpr int NCOL = DVS / 2;           // columns per warp half
  constexpr int CW = NCOL < 32 ? NCOL : 32;   // columns per TMEM load or store
  constexpr int NST = Lay::NST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t *sp = smem_raw + (sb - sraw);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sp + Lay::BAR);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hw = warp >> 2;
  const int unit = blockIdx.x, n = unit / H, h = unit % H;
  const int y = blockIdx.y, col0 = y * DVS;
  const int crow = 32 * qd + lane;

  const int64_t T_n = (int64_t)cu[n + 1] - cu[n];
  const int64_t nch = (T_n + kC - 1) / kC;
  if (!first_window && nch <= jw0) return;   // finished in an earlier window
  const int64_t cnt = window_chunks(cu, n, jw0, wc);

  // First packet of sequence n in this window, and its checkpoint slot.
  if (warp == 0) {
    int64_t before = 0, cks = 0;
    for (int m = lane; m < n; m += 32) {
      before += window_chunks(cu, m, jw0, wc);
      if (interval > 0) cks += ((int64_t)cu[m + 1] - cu[m]) / interval;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, o);
      cks += __shfl_xor_sync(0xffffffffu, cks, o);
    }
    if (lane == 0) {
      reinterpret_cast<int64_t *>(sp + Lay::SCAL)[0] = before;
      if (interval > 0) {
        const int64_t done0 = kC * jw0 < T_n ? kC * jw0 : T_n;
        cks += done0 / interval;
      }
      reinterpret_cast<int64_t *>(sp + Lay::SCAL)[1] = cks;
    }
  }
  uint64_t *sbar = reinterpret_cast<uint64_t *>(sp + Lay::SBAR);
  uint64_t *obar = reinterpret_cast<uint64_t *>(sp + Lay::OBAR);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(sbar, 1);
    mbar_init(obar, 1);
    for (int s = 0; s < NST; ++s) mbar_init(reinterpret_cast<uint64_t *>(sp + Lay::FULL + 8 * s), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tc::tmem_alloc(sb + Lay::TMEM_SLOT, Lay::TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + Lay::TMEM_SLOT);
  const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
  const int64_t before = reinterpret_cast<const int64_t *>(sp + Lay::SCAL)[0];
  int64_t ck_slot = reinterpret_cast<const int64_t *>(sp + Lay::SCAL)[1];

  const uint8_t *pk0 = ws + ((size_t)before * H + (size_t)h * cnt) * Packet::BYTES;
  auto issue = [&](int64_t jl, int s) {
    const uint8_t *pk = pk0 + (size_t)jl * Packet::BYTES;
    const uint32_t st = sb + Lay::STAGE0 + s * Lay::STAGE;
    const uint32_t fb = sb + Lay::FULL + 8 * s;
    mbar_expect_tx(fb, Lay::TX_BYTES);
    bulk_load(st + Lay::WQ, pk + Packet::WQ, 49152, fb);                    // [W; Qtilde] and Khat
    bulk_load(st + Lay::U, pk + Packet::U + (DVS == 128 ? 0 : 8192 * (DVS == 64 ? y : y >> 1)), Lay::UB, fb);
    bulk_load(st + Lay::P, pk + Packet::P, 8704, fb);                       // P and d
  };
  if (tid == 32)
    for (int s = 0; s < NST && s < cnt; ++s) issue(s, s);

  // FP32 state slice in tensor memory (lane c = state row c), BF16 copy in S_T.
  const uint32_t s_tm = tl + Lay::SCOL + hw * NCOL;
  const float *src = first_window ? init : carry;
  {
    const size_t soff = ((size_t)unit * kDK + crow) * kDV + col0 + hw * NCOL;
#pragma unroll
    for (int u = 0; u < NCOL / CW; ++u) {
      float x[CW];
#pragma unroll
      for (int j = 0; j < CW; j += 4) {
        const float4 v4 = src ? *reinterpret_cast<const float4 *>(src + soff + CW * u + j)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        x[j] = v4.x; x[j + 1] = v4.y; x[j + 2] = v4.z; x[j + 3] = v4.w;
      }
      tc::tmem_stw<CW>(s_tm + CW * u, x);
#pragma unroll
      for (int j = 0; j < CW; j += 8)
        st_chunk_s(sp + Lay::S_T + tc::tile_offset(128, crow, (hw * NCOL + CW * u + j) >> 3), x + j);
    }
    tc::tmem_wait_st();
  }
  auto store_state = [&](float *base_ptr, int64_t slot) {
    float *dst = base_ptr + ((size_t)slot * H + h) * kDK * kDV + (size_t)crow * kDV + col0 + hw * NCOL;
#pragma unroll
    for (int u = 0; u < NCOL / CW; ++u) {
      float x[CW];
      tc::tmem_ldw<CW>(s_tm + CW * u, x);
      tc::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < CW; j += 4)
        *reinterpret_cast<float4 *>(dst + CW * u + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
    }
  };
  tc::fence_smem_to_async();
  tc::fence_before_sync();
  __syncthreads();

  int64_t since_ck = interval > 0 ? (kC * jw0) % interval : 0;
  uint32_t phase = 0, sphase = 0, ophase = 0, fphase = 0;   // fphase: bit s = parity of stage s
  bool aborted = false;
  // O of a chunk leaves TMEM while the next chunk's first product runs.
  // Only the four warps on TMEM lanes 64..127 call it: they stage O (bf16) in
  // OBUF, 16-byte chunks of row r permuted by r % 8, then write whole rows.
  constexpr int CH = DVS / 8;   // 16-byte chunks per O row
  constexpr int CHM = (CH < 8 ? CH : 8) - 1;   // chunk permutation mask
  auto write_o = [&](uint32_t acc, int64_t t0, int L) {
    tc::fence_after_sync();
    const int r = 32 * (qd - 2) + lane;
    float a[NCOL];
#pragma unroll
    for (int u = 0; u < NCOL / CW; ++u) tc::tmem_ldw<CW>(tl + acc + hw * NCOL + CW * u, a + CW * u);
    tc::tmem_wait_ld();
#pragma unroll
    for (int cc = 0; cc < NCOL / 8; ++cc) {
      const int c = hw * (NCOL / 8) + cc;
      st_chunk_s(sp + Lay::OBUF + r * (DVS * 2) + ((c ^ (r & CHM)) << 4), a + 8 * cc);
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");   // the four O warps
    const int t = 32 * ((qd - 2) + 2 * hw) + lane;
#pragma unroll
    for (int e = t; e < 64 * CH; e += 128) {
      const int row = e / CH, c = e % CH;
      if (row < L) {
        const uint4 v4 = *reinterpret_cast<const uint4 *>(sp + Lay::OBUF + row * (DVS * 2) + ((c ^ (row & CHM)) << 4));
        *reinterpret_cast<uint4 *>(out + ((size_t)(t0 + row) * H + h) * kDV + col0 + 8 * c) = v4;
      }
    }
  };
  int64_t t0_prev = 0;
  int L_prev = 0;
  int64_t tile_slot = -1;   // a checkpoint to copy out of S_T (BF16 tile mode)
  for (int64_t jl = 0; jl < cnt; ++jl) {
    const int s = (int)(jl % NST);
    const uint32_t st = sb + Lay::STAGE0 + s * Lay::STAGE;
    const uint32_t acc1 = (jl & 1) ? Lay::ACC1B : Lay::ACC1;
    const int64_t j = jw0 + jl;
    const int64_t t0 = cu[n] + kC * j;
    const int L = (int)(T_n - kC * j < kC ? T_n - kC * j : kC);
    if (__syncthreads_or(!wait_timed(reinterpret_cast<uint64_t *>(sp + Lay::FULL + 8 * s),
                                     (fphase >> s) & 1u, wait_ns))) { aborted = true; break; }
    fphase ^= 1u << s;

    // acc1 = [W; Qtilde] S0
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(128, DVS, 0, 1);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        tc::mma_bf16(tmem + acc1, tc::desc_kmajor(st + Lay::WQ, 128, s2),
                     tc::desc_mnmajor(sb + Lay::S_T, 128, s2), id, s2 > 0);
      tc::mma_commit(sb + Lay::BAR);
    }
    if (jl > 0) {
      // The previous chunk's O accumulation is done: its packet buffer may be
      // refilled and its O written out.
      if (__syncthreads_or(!wait_timed(obar, ophase, wait_ns))) { aborted = true; break; }
      ophase ^= 1;
      if (tid == 32 && jl - 1 + NST < cnt) issue(jl - 1 + NST, (int)((jl - 1) % NST));
    }
    // Warps on TMEM lanes 64..127 write the previous chunk's O while the others
    // wait for the first product and form V_new.
    bool late = false;
    if (qd >= 2) {
      if (jl > 0) write_o((jl & 1) ? Lay::ACC1 : Lay::ACC1B, t0_prev, L_prev);
    } else {
      late = !wait_timed(bar, phase, wait_ns);
      tc::fence_after_sync();
      // V_new = U - W S0 (TMEM lanes 0..63), as the bf16 B operand.
      const int r = 32 * qd + lane;
      float a[NCOL];
#pragma unroll
      for (int u = 0; u < NCOL / CW; ++u) tc::tmem_ldw<CW>(tl + acc1 + hw * NCOL + CW * u, a + CW * u);
      tc::tmem_wait_ld();
      const int uc0 = DVS == 32 ? 4 * (y & 1) : 0;   // the slice's first chunk in the U block
#pragma unroll
      for (int cc = 0; cc < NCOL / 8; ++cc) {
        const int chunk = hw * (NCOL / 8) + cc;
        const uint4 uu = *reinterpret_cast<const uint4 *>(sp + (st - sb) + Lay::U + tc::tile_offset(64, r, uc0 + chunk));
        float xv[8];
        unpack8(uu, xv);
#pragma unroll
        for (int e = 0; e < 8; ++e) xv[e] -= a[8 * cc + e];
        st_chunk_s(sp + Lay::VN + tc::tile_offset(64, r, chunk), xv);
      }
    }
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    if (__syncthreads_or(late)) { aborted = true; break; }
    phase ^= 1;

    // acc1 += [*; P] V_new (rows 64..127 become O), acc2 = Khat^T V_new
    if (tid == 0) {
      tc::fence_after_sync();
      constexpr uint32_t ida = tc::idesc_bf16(128, DVS, 0, 1);
      constexpr uint32_t idb = tc::idesc_bf16(128, DVS, 1, 1);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + Lay::ACC2, tc::desc_mnmajor(st + Lay::KH, 64, s2),
                     tc::desc_mnmajor(sb + Lay::VN, 64, s2), idb, s2 > 0);
      tc::mma_commit(sb + Lay::SBAR);
#pragma unroll
      for (int s2 = 0; s2 < 4; ++s2)
        tc::mma_bf16(tmem + acc1, tc::desc_kmajor(st + Lay::P - 8192, 128, s2),
                     tc::desc_mnmajor(sb + Lay::VN, 64, s2), ida, 1);
      tc::mma_commit(sb + Lay::OBAR);
    }
    const float d = reinterpret_cast<const float *>(sp + (st - sb) + Lay::D)[crow];
    if (tid == 32) bulk_wait_read();   // the last checkpoint copy has left S_T
    if (__syncthreads_or(!wait_timed(sbar, sphase, wait_ns))) { aborted = true; break; }
    sphase ^= 1;
    tc::fence_after_sync();
    {
      float a[NCOL], sv[NCOL];
#pragma unroll
      for (int u = 0; u < NCOL / CW; ++u) {
        tc::tmem_ldw<CW>(tl + Lay::ACC2 + hw * NCOL + CW * u, a + CW * u);
        tc::tmem_ldw<CW>(s_tm + CW * u, sv + CW * u);
      }
      tc::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < NCOL; ++i) sv[i] = fmaf(d, sv[i], a[i]);
#pragma unroll
      for (int u = 0; u < NCOL / CW; ++u) tc::tmem_stw<CW>(s_tm + CW * u, sv + CW * u);
#pragma unroll
      for (int jj = 0; jj < NCOL; jj += 8)
        st_chunk_s(sp + Lay::S_T + tc::tile_offset(128, crow, (hw * NCOL + jj) >> 3), sv + jj);
      tc::tmem_wait_st();
      since_ck += L;
      if (interval > 0 && since_ck == interval) {
        if (ck_tiles) tile_slot = ck_slot++;
        else store_state(ck, ck_slot++);
        since_ck = 0;
      }
    }
    t0_prev = t0;
    L_prev = L;
    tc::fence_smem_to_async();
    tc::fence_before_sync();
    __syncthreads();
    if (tile_slot >= 0) {   // the BF16 state tile (this CTA's column block) as the checkpoint
      if (tid == 32) {
        bulk_store(ck_tiles + ((size_t)tile_slot * H + h) * (kDK * kDV * 2) + (size_t)y * (128 * DVS * 2),
                   sb + Lay::S_T, 128 * DVS * 2);
        bulk_commit();
      }
      tile_slot = -1;
    }
  }
  if (tid == 32) bulk_wait_all();
  if (!aborted && cnt > 0) {
    if (__syncthreads_or(!wait_timed(obar, ophase, wait_ns))) aborted = true;
    else {
      ophase ^= 1;
      if (qd >= 2) write_o(((cnt - 1) & 1) ? Lay::ACC1B : Lay::ACC1, t0_prev, L_prev);
    }
  }

  if (aborted) {
    report(dev_status, KDA_ERR_TIMEOUT);
    wait_timed(bar, phase, wait_ns);
    wait_timed(sbar, sphase, wait_ns);
    wait_timed(obar, ophase, wait_ns);
    for (int s = 0; s < NST; ++s)
      wait_timed(reinterpret_cast<uint64_t *>(sp + Lay::FULL + 8 * s), (fphase >> s) & 1u, wait_ns);
  } else if (carry) {
    store_state(carry, n);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

template <int DVS>
cudaError_t launch_chain(const uint8_t *ws, const float *init, const int32_t *cu, void *out,
                         float *carry, int64_t interval, float *ck, uint8_t *ck_tiles, int N, int H,
                         int64_t jw0, int64_t wc, int first, int32_t *dev_status,
                         cudaStream_t stream) {
  const size_t smem = ChainLayout<DVS>::TOTAL + 1024;
  auto kern = chain_kernel<DVS>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)((int64_t)N * H), (unsigned)(kDV / DVS));
  kern<<<grid, kThreads, smem, stream>>>(ws, init, cu, (__nv_bfloat16 *)out, carry, interval, ck,
                                         ck_tiles, N, H, jw0, wc, first, dev_status, 2000000000ull);
  return cudaGetLastError();
}

}  // namespace

// Bytes of one packet (one chunk of one head).
size_t split_packet_bytes() { return Packet::BYTES; }

bool prefill_split_supported(int N) { return N >= 1 && N <= kMaxSeqs; }

// Workspace that runs the whole batch as a single window (an upper bound:
// every sequence may end in a partial chunk), plus the FP32 state carried
// between windows when the caller keeps no final state.
size_t split_workspace_full(int N, int H, int64_t T, bool have_final) {
  const size_t packets = (size_t)H * (size_t)((T + (int64_t)(kC - 1) * N) / kC);
  return packets * Packet::BYTES + (have_final ? 0 : (size_t)N * H * kDK * kDV * 4) + 256;
}

// Two-pass prefill over windows of chunks.  Packets of a window are stored
// sequence by sequence, head by head, chunk by chunk: packet (n, h, j) sits at
// index H * sum_{m<n} c_m + h * c_n + (j - jw0), c_m = chunks of m in the window.
// Checkpoints go to `ck` as FP32 [128][128] states, or, with `ck_tiles` set
// (and `ck` null), as the chain's BF16 state tiles (32 KB each, the 128-byte
// swizzled [key channel][value column] MMA operand layout).  `tt_out` (one
// window only) receives each packet's T and (I + M)^-1 as BF16 tiles.
cudaError_t launch_prefill_split_ex(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const float *init, const int32_t *cu,
                                    void *out, float *fin, int64_t interval, float *ck,
                                    uint8_t *ck_tiles, uint8_t *tt_out, int N, int H, int64_t T,
                                    void *workspace, size_t ws_bytes, int32_t *dev_status,
                                    cudaStream_t stream, int num_sms) {
  if (!prefill_split_supported(N)) return cudaErrorNotSupported;
  uintptr_t base = (reinterpret_cast<uintptr_t>(workspace) + 255) & ~(uintptr_t)255;
  const size_t lost = base - reinterpret_cast<uintptr_t>(workspace);
  if (!workspace || ws_bytes < lost) return cudaErrorInvalidValue;
  size_t avail = ws_bytes - lost;
  const size_t state_bytes = (size_t)N * H * kDK * kDV * 4;
  const int64_t max_chunks = (T + kC - 1) / kC;            // no sequence has more
  const size_t all_packets = (size_t)H * (size_t)((T + (int64_t)(kC - 1) * N) / kC);
  int64_t wc;
  float *carry = fin;
  uint8_t *ws = reinterpret_cast<uint8_t *>(base);
  if (all_packets * Packet::BYTES <= avail) {
    wc = max_chunks > 0 ? max_chunks : 1;                   // one window
  } else {
    if (!fin) {                                             // keep the carried state in the workspace
      if (avail < state_bytes) return cudaErrorInvalidValue;
      avail -= state_bytes;
      carry = reinterpret_cast<float *>(ws + avail);
    }
    wc = (int64_t)(avail / ((size_t)N * H * Packet::BYTES));
    if (wc < 1) return cudaErrorInvalidValue;
  }
  TmaMaps maps;
  if (!make_input_maps(&maps, q, k, v, g, H, T) ||
      !make_map(&maps.q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDK, H, T, 64, 64,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&maps.k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDK, H, T, 64, 64,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem1 = IntraLayout::TOTAL + 1024;
  cudaError_t err = cudaFuncSetAttribute(intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (err != cudaSuccess) return err;
  // Few units: split the value columns over 2 or 4 CTAs per unit (not with
  // state tiles as checkpoints, which a 32-column slice does not fill whole).
  const int slices = ((int64_t)N * H * 4 <= num_sms && !ck_tiles) ? 4 : ((int64_t)N * H * 2 <= num_sms ? 2 : 1);
  const int64_t windows = max_chunks > 0 ? (max_chunks + wc - 1) / wc : 1;
  for (int64_t w = 0; w < windows; ++w) {
    const int64_t jw0 = w * wc;
    if (max_chunks > 0) {
      intra_kernel<<<2 * num_sms, kThreads, smem1, stream>>>(maps, beta, cu, N, H, jw0, wc, ws,
                                                            tt_out, dev_status, 2000000000ull);
      err = cudaGetLastError();
      if (err != cudaSuccess) return err;
    }
    // One window: no carry needed unless the caller wants the final state.
    float *c = (windows == 1) ? fin : carry;
    err = slices == 4 ? launch_chain<32>(ws, init, cu, out, c, interval, ck, ck_tiles, N, H, jw0, wc,
                                         w == 0, dev_status, stream)
        : slices == 2 ? launch_chain<64>(ws, init, cu, out, c, interval, ck, ck_tiles, N, H, jw0, wc,
                                         w == 0, dev_status, stream)
                      : launch_chain<128>(ws, init, cu, out, c, interval, ck, ck_tiles, N, H, jw0, wc,
                                          w == 0, dev_status, stream);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

cudaError_t launch_prefill_split(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *init, const int32_t *cu, void *out,
                                 float *fin, int64_t interval, float *ck, int N, int H, int64_t T,
                                 void *workspace, size_t ws_bytes, int32_t *dev_status,
                                 cudaStream_t stream, int num_sms) {
  return launch_prefill_split_ex(q, k, v, g, beta, init, cu, out, fin, interval, ck, nullptr, nullptr,
                                 N, H, T, workspace, ws_bytes, dev_status, stream, num_sms);
}

}  // namespace kda
