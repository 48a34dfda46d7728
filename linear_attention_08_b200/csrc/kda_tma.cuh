// Copy-engine helpers shared by the tensor-core prefill kernels (sm_100a):
// bounded mbarrier waits on the global timer, 4-byte async copies, TMA tensor
// loads, bulk (non-tensor) copies, and the host-side tensor-map encoder.
#pragma once

#include <cuda.h>

#include "kda_common.cuh"

namespace kda {

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for an mbarrier phase for at most limit_ns nanoseconds.
__device__ __forceinline__ bool wait_timed(uint64_t *bar, uint32_t phase, uint64_t limit_ns) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, phase))
    if (globaltimer() - t0 > limit_ns) return false;
  return true;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Tensor maps of the inputs: 3-D views [T_tot][H][D] of the token-major
// tensors, one box = 64 tokens of one head.
struct TmaMaps {
  CUtensorMap q, k, g, v;
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// Plain bulk copy global -> shared of `bytes` (multiple of 16, both ends
// 16-byte aligned), completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Plain bulk copy shared -> global of `bytes` (multiple of 16, both ends
// 16-byte aligned), tracked by the issuing thread's bulk group.
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The issuing thread's bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// ... and have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Raise the barrier's expected transaction bytes without arriving (a later
// arrive.expect_tx completes the phase's arrival).
__device__ __forceinline__ void mbar_add_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void unpack8(const uint4 &u, float *x) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D map over a token-major tensor [T][H][D]: dims (D, H, T), box
// (box_d, 1, box_t).  Tokens past T read as zeros.
static inline bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt,
                            int elem_bytes, int D, int H, int64_t T, int box_d, int box_t,
                            CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)D * elem_bytes, (cuuint64_t)D * elem_bytes * H};
  const cuuint32_t box[3] = {(cuuint32_t)box_d, 1, (cuuint32_t)box_t};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The four input maps of a 64-token chunk: q, k (bf16, box 128 x 64, rows of
// 256 bytes), g (fp32, box 128 x 64, rows of 512 bytes), v (bf16, box 64 x
// 64, 128-byte swizzle: one column block of an MMA operand tile).
static inline bool make_input_maps(TmaMaps *maps, const void *q, const void *k, const void *v,
                                   const float *g, int H, int64_t T) {
  return make_map(&maps->q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, H, T, 128, 64,
                  CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map(&maps->k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, H, T, 128, 64,
                  CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map(&maps->g, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 128, H, T, 128, 64,
                  CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map(&maps->v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, H, T, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace kda
