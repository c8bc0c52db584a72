// Shared device helpers for libfl (sm_100a): status plumbing, mbarrier and
// bulk-copy PTX, the int8 tensor-core instruction, and the per-group
// fixed-point form of the activation vector used by the int8 products.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <utility>

#include "../../include/fl.h"

namespace fl {

// ---------------------------------------------------------------- host status

void set_error(const char* fmt, ...);
fl_status fail(fl_status st, const char* fmt, ...);
fl_status cuda_fail(cudaError_t e, const char* what);
int device_sm_count();

#define FL_CHECK_CUDA(call, what)                   \
  do {                                              \
    cudaError_t e__ = (call);                       \
    if (e__ != cudaSuccess) return fl::cuda_fail(e__, what); \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- launches
// Every kernel is launched with programmatic stream serialization: the next launch in the
// stream may be scheduled as soon as every CTA of this one has started (pdl_release), and it
// waits (pdl_wait) for this one to finish, memory included, before its first global access.
// Work before the wait (parameter-only set-up) overlaps the previous kernel's tail. Without
// a preceding programmatic launch both are no-ops.
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" :::); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (cluster > 1) {
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = cluster;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- device PTX

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait on an mbarrier phase. Returns false (and leaves the caller to
// record the failure) if the phase has not completed after `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = (1u << 26)) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t k = 0; k < limit; ++k) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// 1-D bulk copy global -> shared (own CTA), completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t rotr32(uint32_t v, uint32_t n) {
  return __funnelshift_r(v, v, n);
}

// D (s32 16x8) += A (u8 16x32, row) * B (s8 32x8, col).
__device__ __forceinline__ void mma_u8s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D (s32 16x8) += A (u8 16x16, row) * B (s8 16x8, col).
__device__ __forceinline__ void mma_u8s8_k16(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// ---------------------------------------------------------------- activations as int8 digits
//
// For the int8 tensor-core products each 128-column group of each activation
// row is written as a 15-bit fixed-point integer  v_c = rint(x_c 2^sigma)
// with sigma = 14 - E, where max_c |x_c| < 2^E, so |v_c| <= 2^14; v_c is then
// split into two balanced signed bytes  v_c = 256 hi_c + lo_c,
// hi_c in [-64, 64], lo_c in [-128, 127].  The group keeps 2^-sigma (to undo
// the scaling) and sum_c v_c (for the constant part of the reconstruction).
// Absolute error per element <= 2^(E - 15) <= 2^-14 max |x_c|. The plane and
// K-quant kernels build these digits in their prologues, each in the shared-memory
// layout its tensor-core fragments read.

}  // namespace fl
