// Merging of logit-gate partials, shared by the gate kernel and the gate fused into the
// batched GEMV. A partial over a set of logits z is (m = max z, S = sum e^(z-m),
// T = sum (z-m) e^(z-m), the top-2 values and indices, ties to the lower index); partials
// merge exactly (up to fp32 rounding) by rescaling S and T to the common maximum.
#pragma once

#include <math.h>

#include "fl_common.cuh"

namespace fl {

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

// Row outputs from a merged partial.
__device__ __forceinline__ void gate_outputs(const GateRec& r, float tau_h, float tau_m, float* entropy, float* margin,
                                             int32_t* top2, uint8_t* escalate) {
  const float H = logf(r.S) - r.T / r.S;
  const float p_gap = (1.0f - expf(r.v2 - r.m)) / r.S;
  *entropy = H;
  *margin = p_gap;
  top2[0] = r.i1;
  top2[1] = r.i2;
  *escalate = (uint8_t)((H > tau_h) || (p_gap < tau_m));
}

}  // namespace fl
