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

// Nanoseconds on the GPU's global timer (advances at wall-clock rate, also while the context
// is switched out).
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Deadline of every wait inside a kernel. A normal wait lasts microseconds; the limit leaves
// room for the context being time-sliced with another process's work.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// One poll of an mbarrier phase. With a suspend-time hint the thread sleeps until the phase
// completes or the hint elapses, instead of returning at once: a waiting warp then takes no
// issue slots from the warps that share its scheduler.
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
               : "=r"(ok)
               : "r"(a), "r"(parity)
               : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_try_sleep(uint32_t a, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(a), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

constexpr uint32_t kSuspendNs = 20000;  // longest single sleep of a waiting thread

// Wait on an mbarrier phase, bounded in time. One plain poll first (the common case in a
// running pipeline); then the thread sleeps in suspend-hinted polls, each ending when the phase
// completes, and the deadline on the global timer is checked between them. Returns false (the
// caller records the failure) if the phase has not completed by then.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_sleep(a, parity, kSuspendNs)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
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

// y += v as a reduction performed in L2 (no value returned, so nothing waits for it); the add
// rounds to nearest like a plain fp32 add.
__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
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
// row is written as a 31-bit fixed-point integer  v_c = rint(x_c 2^sigma)
// with sigma = 30 - E, where max_c |x_c| < 2^E, so |v_c| < 2^30; v_c is then
// split into four balanced signed bytes
//     v_c = 2^24 d3_c + 2^16 d2_c + 2^8 d1_c + d0_c,
// d3_c in [-64, 64], the others in [-128, 127]. A bf16 value has 8
// significant bits, so every element with |x_c| >= 2^-22 max_c |x_c| is
// represented exactly (x_c 2^sigma is then an integer); a smaller element is
// rounded, by at most 2^-sigma / 2 = 2^(E-31) <= 2^-30 of the group's largest |x|.
// The products therefore reproduce sum_c w_c x_c exactly, up to the fp32
// accumulation, unless a group spans more than 22 binades.
//
// The digits enter the products as two pairs per batch row, pair 0 = (d3, d2)
// and pair 1 = (d1, d0); an MMA column pair is one digit pair, so a pair's
// int32 sum is 256 C_hi + C_lo (|C| <= 2^22 per 128 columns, no overflow) and
// weighs 2^16 2^-sigma (pair 0) or 2^-sigma (pair 1). The group keeps both
// weights and 2^-sigma sum_c v_c (for the constant part of the
// reconstruction). The plane and K-quant kernels build these digits in their
// prologues, each in the shared-memory layout its tensor-core fragments read.
//
// split_digits: one warp, 128 columns (four per lane, f[] = this lane's
// values). Writes the lane's four digit words (dw[k] byte i = digit 3-k of
// element i: d3, d2, d1, d0) and the lane's pair sums (part.x = sum of
// 256 d3 + d2, part.y = sum of 256 d1 + d0); returns sigma.
__device__ __forceinline__ int split_digits(const float (&f)[4], uint32_t (&dw)[4], int2& part) {
  uint32_t mb = 0;  // group max |x| (bit patterns of non-negative floats order like the values)
#pragma unroll
  for (int i = 0; i < 4; ++i) mb = max(mb, __float_as_uint(f[i]) & 0x7FFFFFFFu);
  mb = __reduce_max_sync(0xffffffffu, mb);
  int E = 0;  // max |x| = mant * 2^E, mant in [0.5, 1)
  if (mb >= 0x00800000u)
    E = (int)(mb >> 23) - 126;
  else if (mb != 0u)
    frexpf(__uint_as_float(mb), &E);
  const int sigma = (mb != 0u) ? (30 - E) : 0;
  // v = rint(x 2^sigma): a power-of-two scale is exact, so one multiply when 2^sigma is normal
  const bool direct = sigma >= -126 && sigma <= 127;
  const float scale = __uint_as_float((uint32_t)(sigma + 127) << 23);
  dw[0] = dw[1] = dw[2] = dw[3] = 0u;
  part = make_int2(0, 0);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int v = __float2int_rn(direct ? f[i] * scale : ldexpf(f[i], sigma));
    const int h1 = (v + 128) >> 8, d0 = v - 256 * h1;
    const int h2 = (h1 + 128) >> 8, d1 = h1 - 256 * h2;
    const int d3 = (h2 + 128) >> 8, d2 = h2 - 256 * d3;
    dw[0] |= (static_cast<uint32_t>(d3) & 0xFFu) << (8 * i);
    dw[1] |= (static_cast<uint32_t>(d2) & 0xFFu) << (8 * i);
    dw[2] |= (static_cast<uint32_t>(d1) & 0xFFu) << (8 * i);
    dw[3] |= (static_cast<uint32_t>(d0) & 0xFFu) << (8 * i);
    part.x += h2;               // 256 d3 + d2
    part.y += v - 65536 * h2;   // 256 d1 + d0
  }
  return sigma;
}

}  // namespace fl
