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
//
// The same kernel gives the partial of a row piece when the vocabulary is split over devices:
// indices are offset by the piece's first global index and rank 0 stores the merged record
// (max, S, T, top-2) instead of the row's outputs.
#include "fl_gate_merge.cuh"

namespace fl {

__device__ int g_gate_error;  // set if rank 0's wait for the cluster's partials runs out

__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

template <int C, int T, int CACHE, bool PARTIAL>
__global__ void __launch_bounds__(T) logit_gate_kernel(const float* __restrict__ logits, int vocab, float tau_h,
                                                       float tau_m, float* __restrict__ entropy,
                                                       float* __restrict__ margin, int32_t* __restrict__ top2,
                                                       uint8_t* __restrict__ escalate, int index_base,
                                                       GateRec* __restrict__ partial) {
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
  pdl_release();
  pdl_wait();

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
      idx[k] = index_base + 4 * q;
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
    // bounded in time like every other wait (a deadline on the global timer)
    ok = false;
    uint64_t t0 = 0;
    for (uint32_t k = 1; !ok; ++k) {
      uint32_t done;
      asm volatile(
          "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0; selp.u32 %0, 1, 0, p; }"
          : "=r"(done)
          : "r"(smem_u32(&s_bar))
          : "memory");
      ok = done != 0;
      if (ok) break;
      if ((k & 1023u) == 0u) {
        const uint64_t now = globaltimer_ns();
        if (t0 == 0)
          t0 = now;
        else if (now - t0 > kWaitLimitNs)
          break;
      }
    }
    if (!ok) atomicExch(&g_gate_error, 1);
  }
  __syncwarp();
  r = warp_merge(lane < C ? s_cta[lane] : empty_rec());
  if (lane == 0) {
    if constexpr (PARTIAL) {
      if (!ok) r.S = NAN;  // the merged gate's entropy and margin come out NaN
      partial[row] = r;
    } else {
      gate_outputs(r, tau_h, tau_m, entropy + row, margin + row, top2 + 2 * row, escalate + row);
      if (!ok) entropy[row] = margin[row] = NAN;
    }
  }
}

}  // namespace fl

namespace fl {

template <int C, int T, int CACHE, bool PARTIAL>
static cudaError_t gate_launch_c(const float* logits, int vocab, int batch, float tau_h, float tau_m, float* entropy,
                                 float* margin, int32_t* top2, uint8_t* escalate, int index_base, GateRec* partial,
                                 cudaStream_t st) {
  return launch_pdl(logit_gate_kernel<C, T, CACHE, PARTIAL>, dim3((unsigned)(batch * C)), dim3(T), 0, st, C, logits,
                    vocab, tau_h, tau_m, entropy, margin, top2, escalate, index_base, partial);
}

// 16-CTA clusters where the device can place one (decided once per process), else 8.
static bool gate_wide_clusters() {
  static int wide = -1;
  if (wide < 0) {
    auto kern = logit_gate_kernel<16, 256, 10, false>;
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
    return gate_launch_c<16, 256, 10, false>(logits, vocab, batch, tau_h, tau_m, entropy, margin, top2, escalate, 0,
                                             nullptr, st);
  return gate_launch_c<8, 512, 10, false>(logits, vocab, batch, tau_h, tau_m, entropy, margin, top2, escalate, 0,
                                          nullptr, st);
}

// The partial records of the rows' pieces (indices offset by index_base), one cluster per row.
cudaError_t gate_partial_launch(const float* logits, int vocab, int batch, int index_base, GateRec* partial,
                                cudaStream_t st) {
  if (gate_wide_clusters()) {
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(logit_gate_kernel<16, 256, 10, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      attr = true;
    }
    return gate_launch_c<16, 256, 10, true>(logits, vocab, batch, 0.f, 0.f, nullptr, nullptr, nullptr, nullptr,
                                            index_base, partial, st);
  }
  return gate_launch_c<8, 512, 10, true>(logits, vocab, batch, 0.f, 0.f, nullptr, nullptr, nullptr, nullptr,
                                         index_base, partial, st);
}

}  // namespace fl

namespace fl {

// Reads and clears the error word (-1 if that fails).
int take_gate_error() {
  int v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_gate_error, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0 && cudaMemcpyToSymbol(g_gate_error, &z, sizeof(int)) != cudaSuccess) return -1;
  return v;
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
  if ((reinterpret_cast<uintptr_t>(entropy) | reinterpret_cast<uintptr_t>(margin) | reinterpret_cast<uintptr_t>(top2)) &
      3u)
    return fail(FL_ERR_ALIGN, "%s: entropy, margin and top2 must be 4-byte aligned", what);
  FL_CHECK_CUDA(gate_launch(logits, vocab, batch, tau_h, tau_m, entropy, margin, top2, escalate,
                            static_cast<cudaStream_t>(stream)),
                "launch logit_gate");
  return FL_OK;
}
