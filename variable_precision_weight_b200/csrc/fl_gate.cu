// Logit uncertainty gate ("Precision on Demand: Escalating Weight Bits at
// Uncertain Decoding Steps in a Small Local Model", abstract: redo a step at
// 8 bits only when the low-precision output distribution looks uncertain,
// entropy above a threshold or a small top-two margin).
//
// Per logit row t:  m = max z,  S = sum e^(z-m),  T = sum (z-m) e^(z-m),
//   entropy = ln S - T / S,  margin = p1 - p2 = (1 - e^(z_i2 - m)) / S,
//   escalate = entropy > tau_h || margin < tau_m,
// with i1, i2 the two largest logits (ties to the lower index).
//
// One thread-block cluster of C CTAs per row (16 where the GPU can co-schedule that many,
// else 8), each CTA an equal slice of the row held in registers (16-byte loads issued up
// front). Each thread takes the top-2 of its values and S, T relative to its own max; the
// partials (max, S, T, top-2) merge within a warp with redux max/min for the max and the
// top-2 and shuffles for the rescaled sums, then across warps through shared memory, then
// across the cluster: every CTA stores its partial into CTA rank 0's shared memory and
// arrives on an mbarrier there, and rank 0 merges and writes the row's outputs. Merge orders
// are fixed (deterministic); one launch, no global scratch.
#include <math.h>

#include "fl_common.cuh"

namespace fl {

__device__ int g_gate_error;  // set if rank 0's wait for the cluster's partials runs out

struct __align__(16) GateRec {
  float m, S, T, v2;  // max, sum e^(z-m), sum (z-m) e^(z-m), second largest value
  int i1, i2, pad0, pad1;  // indices of the largest and second largest (ties to the lower index)
};

__device__ __forceinline__ bool better(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

struct Top2 {
  float v1, v2;
  int i1, i2;
};

__device__ __forceinline__ void push_top2(Top2& a, float v, int i) {
  if (better(v, i, a.v2, a.i2)) {
    if (better(v, i, a.v1, a.i1)) {
      a.v2 = a.v1;
      a.i2 = a.i1;
      a.v1 = v;
      a.i1 = i;
    } else {
      a.v2 = v;
      a.i2 = i;
    }
  }
}

// Order-preserving map of a float onto uint32 (for redux max).
__device__ __forceinline__ uint32_t okey(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float from_okey(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ GateRec empty_rec() {
  GateRec r;
  r.m = r.v2 = -INFINITY;
  r.S = r.T = 0.f;
  r.i1 = r.i2 = 0x7fffffff;
  r.pad0 = r.pad1 = 0;
  return r;
}

// Merge the 32 lanes' partials; every lane gets the result.
__device__ __forceinline__ GateRec warp_merge(const GateRec& r) {
  const unsigned full = 0xffffffffu;
  GateRec o;
  o.m = from_okey(__reduce_max_sync(full, okey(r.m)));
  o.i1 = __reduce_min_sync(full, (r.m == o.m) ? r.i1 : 0x7fffffff);
  // second: the winner lane offers its own second, every other lane its first
  const bool win = (r.m == o.m) && (r.i1 == o.i1);
  const float cv = win ? r.v2 : r.m;
  const int ci = win ? r.i2 : r.i1;
  o.v2 = from_okey(__reduce_max_sync(full, okey(cv)));
  o.i2 = __reduce_min_sync(full, (cv == o.v2) ? ci : 0x7fffffff);
  // sums rescaled to the common max
  float S = 0.f, T = 0.f;
  if (r.S > 0.f) {
    const float d = r.m - o.m, f = __expf(d);
    S = r.S * f;
    T = fmaf(d, r.S, r.T) * f;
  }
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) {
    S += __shfl_xor_sync(full, S, k);
    T += __shfl_xor_sync(full, T, k);
  }
  o.S = S;
  o.T = T;
  o.pad0 = o.pad1 = 0;
  return o;
}

// Partial of one thread's values z (count n, first index i0 + 4 k + c for float4 k).
template <int CACHE>
__device__ __forceinline__ GateRec thread_partial(const float4 (&v)[CACHE], const int (&idx)[CACHE], int nv) {
  Top2 a;
  a.v1 = a.v2 = -INFINITY;
  a.i1 = a.i2 = 0x7fffffff;
#pragma unroll
  for (int k = 0; k < CACHE; ++k) {
    if (k < nv) {
      push_top2(a, v[k].x, idx[k]);
      push_top2(a, v[k].y, idx[k] + 1);
      push_top2(a, v[k].z, idx[k] + 2);
      push_top2(a, v[k].w, idx[k] + 3);
    }
  }
  GateRec r = empty_rec();
  r.m = a.v1;
  r.v2 = a.v2;
  r.i1 = a.i1;
  r.i2 = a.i2;
  if (nv > 0) {
    float S = 0.f, T = 0.f;
#pragma unroll
    for (int k = 0; k < CACHE; ++k) {
      if (k < nv) {
        const float z[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float d = z[c] - a.v1, e = __expf(d);
          S += e;
          T = fmaf(d, e, T);
        }
      }
    }
    r.S = S;
    r.T = T;
  }
  return r;
}

// Merge two partials (used only when a thread's slice does not fit its registers).
__device__ __forceinline__ GateRec merge2(const GateRec& a, const GateRec& b) {
  GateRec o = a;
  Top2 t;
  t.v1 = a.m;
  t.i1 = a.i1;
  t.v2 = a.v2;
  t.i2 = a.i2;
  push_top2(t, b.m, b.i1);
  push_top2(t, b.v2, b.i2);
  o.m = t.v1;
  o.i1 = t.i1;
  o.v2 = t.v2;
  o.i2 = t.i2;
  float S = 0.f, T = 0.f;
  if (a.S > 0.f) {
    const float d = a.m - o.m, f = __expf(d);
    S += a.S * f;
    T += fmaf(d, a.S, a.T) * f;
  }
  if (b.S > 0.f) {
    const float d = b.m - o.m, f = __expf(d);
    S += b.S * f;
    T += fmaf(d, b.S, b.T) * f;
  }
  o.S = S;
  o.T = T;
  return o;
}

__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

template <int C, int T, int CACHE>
__global__ void __launch_bounds__(T) logit_gate_kernel(const float* __restrict__ logits, int vocab, float tau_h,
                                                       float tau_m, float* __restrict__ entropy,
                                                       float* __restrict__ margin, int32_t* __restrict__ top2,
                                                       uint8_t* __restrict__ escalate) {
  __shared__ GateRec s_warp[T / 32];
  __shared__ GateRec s_cta[C];          // used in rank 0: one slot per CTA of the cluster
  __shared__ __align__(8) uint64_t s_bar;  // rank 0: the other CTAs' partials have arrived
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const int row = blockIdx.x / C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (rank == 0 && threadIdx.x == 0) {
    mbar_init(&s_bar, C - 1);
    fence_mbar_init();
  }
  // every thread arrives once; the other CTAs' senders wait on it before touching rank 0
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");

  const float4* z4 = reinterpret_cast<const float4*>(logits + (size_t)row * vocab);
  const int n4 = vocab / 4;
  const int per = (n4 + C - 1) / C;
  const int q0s = min(n4, (int)rank * per), q1 = min(n4, q0s + per);

  GateRec r = empty_rec();
  for (int base = q0s; base < q1; base += T * CACHE) {
    float4 v[CACHE];
    int idx[CACHE];
    int nv = 0;
#pragma unroll
    for (int k = 0; k < CACHE; ++k) {
      const int q = base + (int)threadIdx.x + k * T;
      idx[k] = 4 * q;
      if (q < q1) {
        v[k] = __ldg(z4 + q);
        nv = k + 1;
      } else {
        v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const GateRec p = thread_partial<CACHE>(v, idx, nv);
    r = (base == q0s) ? p : merge2(r, p);
  }

  // warp, then CTA
  r = warp_merge(r);
  if (lane == 0) s_warp[warp] = r;
  __syncthreads();
  if (warp != 0) return;
  r = warp_merge(lane < T / 32 ? s_warp[lane] : empty_rec());

  // cluster: partials into rank 0's slots
  if (rank != 0) {
    if (lane == 0) {
      asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
      const uint32_t dst = mapa(smem_u32(&s_cta[rank]), 0);
      asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "f"(r.m), "f"(r.S), "f"(r.T),
                   "f"(r.v2)
                   : "memory");
      asm volatile("st.shared::cluster.v2.s32 [%0], {%1, %2};" ::"r"(dst + 16u), "r"(r.i1), "r"(r.i2) : "memory");
      const uint32_t bar = mapa(smem_u32(&s_bar), 0);
      asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
    }
    return;
  }
  if (lane == 0) s_cta[0] = r;
  bool ok = true;
  if (lane == 0) {
    ok = false;
    for (uint32_t k = 0; k < (1u << 24) && !ok; ++k) {
      uint32_t done;
      asm volatile(
          "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0; selp.u32 %0, 1, 0, p; }"
          : "=r"(done)
          : "r"(smem_u32(&s_bar))
          : "memory");
      ok = done != 0;
    }
    if (!ok) atomicExch(&g_gate_error, 1);
  }
  __syncwarp();
  r = warp_merge(lane < C ? s_cta[lane] : empty_rec());
  if (lane == 0) {
    const float H = logf(r.S) - r.T / r.S;
    const float p_gap = (1.0f - expf(r.v2 - r.m)) / r.S;
    entropy[row] = ok ? H : NAN;
    margin[row] = ok ? p_gap : NAN;
    top2[2 * row] = r.i1;
    top2[2 * row + 1] = r.i2;
    escalate[row] = (uint8_t)((H > tau_h) || (p_gap < tau_m));
  }
}

}  // namespace fl

namespace fl {

template <int C, int T, int CACHE>
static cudaError_t gate_launch_c(const float* logits, int vocab, int batch, float tau_h, float tau_m, float* entropy,
                                 float* margin, int32_t* top2, uint8_t* escalate, cudaStream_t st) {
  auto kern = logit_gate_kernel<C, T, CACHE>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(batch * C));
  cfg.blockDim = dim3(T);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, logits, vocab, tau_h, tau_m, entropy, margin, top2, escalate);
}

// 16-CTA clusters where the device can place one (decided once per process), else 8.
static bool gate_wide_clusters() {
  static int wide = -1;
  if (wide < 0) {
    auto kern = logit_gate_kernel<16, 256, 10>;
    int n = 0;
    bool ok = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    if (ok) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16);
      cfg.blockDim = dim3(256);
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 16;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      ok = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0;
    }
    cudaGetLastError();  // a refused query leaves no sticky error
    wide = ok ? 1 : 0;
  }
  return wide == 1;
}

static cudaError_t gate_launch(const float* logits, int vocab, int batch, float tau_h, float tau_m, float* entropy,
                               float* margin, int32_t* top2, uint8_t* escalate, cudaStream_t st) {
  if (gate_wide_clusters())
    return gate_launch_c<16, 256, 10>(logits, vocab, batch, tau_h, tau_m, entropy, margin, top2, escalate, st);
  return gate_launch_c<8, 512, 10>(logits, vocab, batch, tau_h, tau_m, entropy, margin, top2, escalate, st);
}

}  // namespace fl

extern "C" fl_status fl_logit_gate(const float* logits, int vocab, int batch, float tau_h, float tau_m,
                                   float* entropy, float* margin, int32_t* top2, uint8_t* escalate, void* stream) {
  using namespace fl;
  const char* what = "fl_logit_gate";
  if (!logits || !entropy || !margin || !top2 || !escalate) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  if (vocab < 4 || vocab > (1 << 24) || vocab % 4) return fail(FL_ERR_SHAPE, "%s: vocab=%d (4..2^24, %% 4 == 0)", what, vocab);
  if (!aligned16(logits)) return fail(FL_ERR_ALIGN, "%s: logits not 16-byte aligned", what);
  FL_CHECK_CUDA(gate_launch(logits, vocab, batch, tau_h, tau_m, entropy, margin, top2, escalate,
                            static_cast<cudaStream_t>(stream)),
                "launch logit_gate");
  return FL_OK;
}
