// Lens level map ("Precision where the question is, not everywhere", section
// "The mechanism", rules 1-7).
//
// One thread per block. For every lens: R_i = r_i f / (1 - f), Euclidean
// distance to the centre, rho_i = d / R_i, L_i = max(0, 1 - rho_i / s_last);
// combine by clamped sum or by max; rho* = s_last (1 - L); the level is
// gamma plus the number of stops strictly above rho* (ring j covers
// [s_(j+1), s_j), s_(kappa+1) = 0), so a block outside every lens (L = 0,
// rho* = s_last) sits at gamma. Every operation is an explicitly rounded fp32
// intrinsic in that fixed order, so no multiply-add is fused and the levels
// are reproducible bit for bit. Lens data sit in shared memory; per-level
// counts are reduced in shared memory and added to the caller's counters.
#include <math.h>

#include "fl_common.cuh"

namespace fl {

struct LensArgs {
  float f;
  int gamma;
  int kappa;
  int nstops;
  int combine;
  int nlenses;
  int nlevels;
  float stops[FL_MAX_STOPS];
};

__global__ void __launch_bounds__(256) level_map_kernel(const float* __restrict__ xy, int nblocks,
                                                        const float* __restrict__ centers,
                                                        const float* __restrict__ radii, LensArgs a,
                                                        uint8_t* __restrict__ levels, uint32_t* __restrict__ counts) {
  __shared__ float s_cx[64], s_cy[64], s_R[64];
  __shared__ uint32_t s_cnt[16];
  pdl_release();
  pdl_wait();
  if (threadIdx.x < 16) s_cnt[threadIdx.x] = 0;
  if (threadIdx.x < a.nlenses) {
    const float num = __fmul_rn(radii[threadIdx.x], a.f);
    const float den = __fsub_rn(1.0f, a.f);
    s_R[threadIdx.x] = __fdiv_rn(num, den);
    s_cx[threadIdx.x] = centers[2 * threadIdx.x];
    s_cy[threadIdx.x] = centers[2 * threadIdx.x + 1];
  }
  __syncthreads();
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += gridDim.x * blockDim.x) {
    int lev = a.gamma;
    if (a.kappa > a.gamma && a.nlenses > 0) {
      const float s_last = a.stops[a.nstops - 1];
      const float bx = xy[2 * b], by = xy[2 * b + 1];
      float L = 0.0f;
      for (int i = 0; i < a.nlenses; ++i) {
        const float dx = __fsub_rn(bx, s_cx[i]);
        const float dy = __fsub_rn(by, s_cy[i]);
        const float d = __fsqrt_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)));
        const float R = s_R[i];
        float rho;
        if (R > 0.0f)
          rho = __fdiv_rn(d, R);
        else
          rho = (d == 0.0f) ? 0.0f : INFINITY;
        float li = __fsub_rn(1.0f, __fdiv_rn(rho, s_last));
        if (!(li > 0.0f)) li = 0.0f;
        if (a.combine == 0)
          L = __fadd_rn(L, li);
        else if (li > L)
          L = li;
      }
      if (L > 1.0f) L = 1.0f;
      const float rho_star = __fmul_rn(s_last, __fsub_rn(1.0f, L));
      for (int j = 0; j < a.nstops; ++j)
        if (rho_star < a.stops[j]) ++lev;
    }
    levels[b] = static_cast<uint8_t>(lev);
    if (counts) atomicAdd(&s_cnt[lev], 1u);
  }
  if (counts) {
    __syncthreads();
    if (threadIdx.x < a.nlevels && s_cnt[threadIdx.x]) atomicAdd(&counts[threadIdx.x], s_cnt[threadIdx.x]);
  }
}

}  // namespace fl

extern "C" fl_status fl_level_map(const float* xy, int nblocks, const float* centers, const float* radii,
                                  int nlenses, const fl_lens_params* p, uint8_t* levels, uint32_t* counts,
                                  void* stream) {
  using namespace fl;
  const char* what = "fl_level_map";
  if (!p) return fail(FL_ERR_ARG, "%s: params is NULL", what);
  if (nblocks < 0 || nlenses < 0 || nlenses > 64) return fail(FL_ERR_ARG, "%s: nblocks=%d nlenses=%d", what, nblocks, nlenses);
  if (nblocks > 0 && (!xy || !levels)) return fail(FL_ERR_ARG, "%s: NULL xy/levels", what);
  if (nlenses > 0 && (!centers || !radii)) return fail(FL_ERR_ARG, "%s: NULL centers/radii", what);
  if ((reinterpret_cast<uintptr_t>(xy) | reinterpret_cast<uintptr_t>(centers) | reinterpret_cast<uintptr_t>(radii) |
       reinterpret_cast<uintptr_t>(counts)) & 3u)
    return fail(FL_ERR_ALIGN, "%s: xy, centers, radii and counts must be 4-byte aligned", what);
  if (p->m < 1 || p->m > 15 || p->gamma < 0 || p->gamma > p->m)
    return fail(FL_ERR_ARG, "%s: gamma=%d m=%d", what, p->gamma, p->m);
  if (!(p->f >= 0.0f && p->f < 1.0f)) return fail(FL_ERR_ARG, "%s: f=%g (0 <= f < 1)", what, (double)p->f);
  if (!(p->g >= 0.0f && p->g <= 1.0f)) return fail(FL_ERR_ARG, "%s: g=%g (0 <= g <= 1)", what, (double)p->g);
  if (p->combine != 0 && p->combine != 1) return fail(FL_ERR_ARG, "%s: combine=%d", what, p->combine);
  const float t = p->g * (float)(p->m - p->gamma);
  const int kappa = p->gamma + (int)floorf(t);
  if (p->nstops != kappa - p->gamma)
    return fail(FL_ERR_ARG, "%s: nstops=%d but kappa - gamma = %d", what, p->nstops, kappa - p->gamma);
  if (p->nstops > FL_MAX_STOPS) return fail(FL_ERR_ARG, "%s: too many stops", what);
  for (int j = 0; j < p->nstops; ++j) {
    if (!(p->stops[j] > 0.0f) || (j > 0 && !(p->stops[j] > p->stops[j - 1])))
      return fail(FL_ERR_ARG, "%s: stops must be positive and strictly ascending", what);
  }
  if (nblocks == 0) return FL_OK;
  LensArgs a;
  a.f = p->f;
  a.gamma = p->gamma;
  a.kappa = kappa;
  a.nstops = p->nstops;
  a.combine = p->combine;
  a.nlenses = nlenses;
  a.nlevels = p->m + 1;
  for (int j = 0; j < FL_MAX_STOPS; ++j) a.stops[j] = j < p->nstops ? p->stops[j] : 0.0f;
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  int grid = (nblocks + 255) / 256;
  if (grid > nsm * 4) grid = nsm * 4;
  FL_CHECK_CUDA(launch_pdl(level_map_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), 1, xy,
                           nblocks, centers, radii, a, levels, counts),
                "launch level_map");
  return FL_OK;
}
