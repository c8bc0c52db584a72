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
// One thread-block cluster of kClusterCtas CTAs per row: every CTA streams an
// equal slice of the row with 16-byte loads, keeping an online
// (max, S, T, top-2) per thread; partials are merged with warp shuffles, then
// across warps in shared memory, then across the cluster through distributed
// shared memory by CTA rank 0, which writes the row's outputs. One launch, no
// global scratch, no atomics, fixed merge order (deterministic).
#include <cooperative_groups.h>
#include <math.h>

#include "fl_common.cuh"

namespace cg = cooperative_groups;

namespace fl {

constexpr int kClusterCtas = 8;
constexpr int kGateThreads = 1024;
constexpr int kGateUnroll = 8;  // float4 loads in flight per thread

struct GateAcc {
  float m, S, T;   // running max, sum e^(z-m), sum (z-m) e^(z-m)
  float v1, v2;    // top-2 values
  int i1, i2;      // top-2 indices
};

__device__ __forceinline__ bool better(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

__device__ __forceinline__ void push_top2(GateAcc& a, float v, int i) {
  if (better(v, i, a.v1, a.i1)) {
    a.v2 = a.v1;
    a.i2 = a.i1;
    a.v1 = v;
    a.i1 = i;
  } else if (better(v, i, a.v2, a.i2)) {
    a.v2 = v;
    a.i2 = i;
  }
}

__device__ __forceinline__ void merge(GateAcc& a, const GateAcc& b) {
  const float m = fmaxf(a.m, b.m);
  float S = 0.f, T = 0.f;
  if (a.S > 0.f) {
    const float ea = expf(a.m - m);
    S += a.S * ea;
    T += (a.T + (a.m - m) * a.S) * ea;
  }
  if (b.S > 0.f) {
    const float eb = expf(b.m - m);
    S += b.S * eb;
    T += (b.T + (b.m - m) * b.S) * eb;
  }
  a.m = m;
  a.S = S;
  a.T = T;
  push_top2(a, b.v1, b.i1);
  push_top2(a, b.v2, b.i2);
}

__device__ __forceinline__ GateAcc shfl_acc(const GateAcc& a, int src_lane_xor) {
  GateAcc b;
  b.m = __shfl_xor_sync(0xffffffffu, a.m, src_lane_xor);
  b.S = __shfl_xor_sync(0xffffffffu, a.S, src_lane_xor);
  b.T = __shfl_xor_sync(0xffffffffu, a.T, src_lane_xor);
  b.v1 = __shfl_xor_sync(0xffffffffu, a.v1, src_lane_xor);
  b.v2 = __shfl_xor_sync(0xffffffffu, a.v2, src_lane_xor);
  b.i1 = __shfl_xor_sync(0xffffffffu, a.i1, src_lane_xor);
  b.i2 = __shfl_xor_sync(0xffffffffu, a.i2, src_lane_xor);
  return b;
}

__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kGateThreads)
    logit_gate_kernel(const float* __restrict__ logits, int vocab, float tau_h, float tau_m,
                      float* __restrict__ entropy, float* __restrict__ margin, int32_t* __restrict__ top2,
                      uint8_t* __restrict__ escalate) {
  __shared__ GateAcc s_warp[kGateThreads / 32];
  __shared__ GateAcc s_cta;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / kClusterCtas;
  const float* z = logits + (size_t)row * vocab;

  // this CTA's slice, in float4 units
  const int n4 = vocab / 4;
  const int per = (n4 + kClusterCtas - 1) / kClusterCtas;
  const int q0s = rank * per, q1 = min(n4, q0s + per);

  GateAcc a;
  a.m = -INFINITY;
  a.S = 0.f;
  a.T = 0.f;
  a.v1 = a.v2 = -INFINITY;
  a.i1 = a.i2 = 0x7fffffff;
  // All of a thread's 16-byte loads are issued before any is used (a row slice is at most
  // kGateUnroll float4 per thread for the vocabularies in use; longer rows loop).
  for (int q0 = q0s + (int)threadIdx.x; q0 < q1; q0 += kGateThreads * kGateUnroll) {
    float4 v[kGateUnroll];
#pragma unroll
    for (int k = 0; k < kGateUnroll; ++k) {
      const int q = q0 + k * kGateThreads;
      v[k] = (q < q1) ? __ldg(reinterpret_cast<const float4*>(z) + q) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    float mx = a.m;
#pragma unroll
    for (int k = 0; k < kGateUnroll; ++k) mx = fmaxf(mx, fmaxf(fmaxf(v[k].x, v[k].y), fmaxf(v[k].z, v[k].w)));
    if (mx > a.m) {
      if (a.S > 0.f) {
        const float r = expf(a.m - mx);
        a.T = (a.T + (a.m - mx) * a.S) * r;
        a.S = a.S * r;
      }
      a.m = mx;
    }
#pragma unroll
    for (int k = 0; k < kGateUnroll; ++k) {
      const int q = q0 + k * kGateThreads;
      if (q < q1) {
        const float e[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float dz = e[c] - a.m;
          const float ex = expf(dz);
          a.S += ex;
          a.T += dz * ex;
          push_top2(a, e[c], 4 * q + c);
        }
      }
    }
  }
  // warp, then CTA
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    GateAcc b = shfl_acc(a, o);
    merge(a, b);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_warp[warp] = a;
  __syncthreads();
  if (warp == 0) {  // the 32 warp partials, merged by warp 0 with shuffles
    GateAcc c = s_warp[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      GateAcc b = shfl_acc(c, o);
      merge(c, b);
    }
    if (lane == 0) s_cta = c;
  }
  cluster.sync();
  if (rank == 0 && threadIdx.x == 0) {
    GateAcc c = s_cta;
    for (int r = 1; r < kClusterCtas; ++r) {
      const GateAcc* other = cluster.map_shared_rank(&s_cta, r);
      merge(c, *other);
    }
    const float H = logf(c.S) - c.T / c.S;
    const float p_gap = (1.0f - expf(c.v2 - c.m)) / c.S;
    entropy[row] = H;
    margin[row] = p_gap;
    top2[2 * row] = c.i1;
    top2[2 * row + 1] = c.i2;
    escalate[row] = (uint8_t)((H > tau_h) || (p_gap < tau_m));
  }
  cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
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
  logit_gate_kernel<<<batch * kClusterCtas, kGateThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      logits, vocab, tau_h, tau_m, entropy, margin, top2, escalate);
  FL_CHECK_CUDA(cudaGetLastError(), "launch logit_gate");
  return FL_OK;
}
