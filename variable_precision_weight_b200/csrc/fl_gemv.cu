// Depth-dispatched bit-plane GEMV / skinny GEMM and the escalation residual.
//
// What it computes ("FoQLens" landing page, progress table: every block of
// rows read to its own depth straight from the stored copy; "Precision on
// Demand", abstract: decode with the top bits, redo at 8 bits):
//   depth mode     y[t][r]  = sum_c s[r][c/128] (u_d - 128 + c_d) x[t][c]
//   residual mode  y[t][r] += sum_c s[r][c/128] ((u_b - u_a) + c_b - c_a) x[t][c]
// with u_d the top d bits of u = code + 128 kept in place, c_d = (2^(8-d)-1)/2
// and c_0 := 128, u_0 := 0 (the ZERO level contributes nothing).
//
// How (B200): one persistent CTA per SM, warp-specialised.
//  * A producer warp walks the CTA's contiguous range of work units
//    (problem, column slice, 64-row block) and, per tile of whole 128-column
//    groups, issues 1-D bulk copies of the block's scales and of the planes
//    the block's depth needs (a contiguous span per plane in the store) into
//    a 4-stage shared-memory ring guarded by mbarriers. Planes the depth does
//    not need are never fetched.
//  * Eight consumer warps (4 m-tiles of 16 rows x 2 group parities) assemble,
//    per 16 columns, the code bytes u_d from the plane words with one AND/OR
//    per plane and one rotate (the store layout places each plane's field so
//    that this yields u_d in byte lanes), and feed them as the u8 operand of
//    mma.sync m16n8k32 against the activations written as two signed int8
//    digits of a 15-bit per-group fixed point. Integer sums per 128-column
//    group are turned into fp32 with the group scale and the constant part
//    (c_d - 128) sum_c x_c, then accumulated in fp32.
//  * When a layer has too few blocks to fill the GPU its columns are split
//    into slices; each slice writes a partial to the caller's workspace and
//    the last CTA to finish a block (an atomic ticket) adds the partials in
//    slice order, so results are deterministic. No CTA ever waits on another.
#include <algorithm>
#include <vector>

#include "fl_common.cuh"

namespace fl {
namespace gemv {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kStages = 4;
constexpr int kStageBytes = 36864;
constexpr int kMaxCtas = 512;
constexpr int kSmemLimit = 232448 - 6144;  // opt-in shared memory per block on B200, less static use

// Groups per tile for a given number of planes: largest tg with
// tg * (256 + 2048 np) <= kStageBytes.
__host__ __device__ constexpr int tile_groups(int np) {
  return np == 1 ? 16 : np == 2 ? 8 : np == 3 ? 5 : 4;
}

struct Problem {
  const uint8_t* store;
  const uint8_t* lv_from;
  const uint8_t* lv_to;
  const uint16_t* x;
  float* y;
  float* partial;      // [slices][nblocks][batch][64] when slices > 1
  uint32_t* tickets;   // [nblocks] when slices > 1
  int nblocks;
  int G;
  int slices;
  int slice_groups;    // groups per slice (last slice shorter)
  int unit_begin;      // first global unit index of this problem
};

template <int MAXP>
struct Args {
  int nproblems;
  int batch;
  int mode;            // 0 depth (y =), 1 residual (y +=)
  int digit_stride;    // bytes per digit row in smem
  int max_slice_groups;
  int ncta;
  int cta_begin[kMaxCtas + 1];
  Problem p[MAXP];
};

__device__ int g_error;  // set on a bounded wait that ran out (never expected)

struct UnitCursor {
  int p, j, b, u;  // problem, slice, block, global unit
};

template <int MAXP>
__device__ __forceinline__ UnitCursor cursor_at(const Args<MAXP>& a, int u) {
  int p = 0;
  while (p + 1 < a.nproblems && a.p[p + 1].unit_begin <= u) ++p;
  const int local = u - a.p[p].unit_begin;
  UnitCursor c;
  c.p = p;
  c.j = local / a.p[p].nblocks;
  c.b = local % a.p[p].nblocks;
  c.u = u;
  return c;
}

template <int MAXP>
__device__ __forceinline__ void cursor_next(const Args<MAXP>& a, UnitCursor& c) {
  ++c.u;
  if (++c.b == a.p[c.p].nblocks) {
    c.b = 0;
    if (++c.j == a.p[c.p].slices) {
      c.j = 0;
      ++c.p;
    }
  }
}

// Plane range [k0, k0 + np) read for a block.
template <int MAXP>
__device__ __forceinline__ void plane_range(const Args<MAXP>& a, const Problem& P, int b, int& k0, int& np) {
  int lf = min((int)P.lv_from[b], 4);
  if (a.mode == 0) {
    k0 = 0;
    np = lf;
  } else {
    int lt = min((int)P.lv_to[b], 4);
    k0 = lf;
    np = max(0, lt - lf);
  }
}

__device__ __forceinline__ int slice_g0(const Problem& P, int j) { return j * P.slice_groups; }
__device__ __forceinline__ int slice_ng(const Problem& P, int j) {
  return min(P.slice_groups, P.G - j * P.slice_groups);
}

// Mask selecting plane k's fields for column set i (rotl(0x03030303, 6-2k+2i)).
__host__ __device__ constexpr uint32_t plane_mask(int k, int i) {
  return (((6 - 2 * k + 2 * i) & 7) == 0)
             ? 0x03030303u
             : ((0x03030303u << ((6 - 2 * k + 2 * i) & 7)) | (0x03030303u >> (32 - ((6 - 2 * k + 2 * i) & 7))));
}

// One 128-column group for one m-tile: 4 k32 MMAs per N-tile.
// W[kk][r][w]: word w (0,1) of row r (0: g, 1: g + 8) of plane k0 + kk.
template <int K0, int NP, int NT>
__device__ __forceinline__ void group_mma(const uint2 (&W)[4][2], const uint4 (&B)[NT][2], int32_t (&C)[NT][4]) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int w = s >> 1;
    const int i0 = 2 * (s & 1), i1 = i0 + 1;
    uint32_t u[2][2];  // [row][i0/i1]
#pragma unroll
    for (int r = 0; r < 2; ++r) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = h ? i1 : i0;
        uint32_t acc = 0;
#pragma unroll
        for (int kk = 0; kk < NP; ++kk) {
          const uint32_t word = w ? W[kk][r].y : W[kk][r].x;
          acc |= word & plane_mask(K0 + kk, i);
        }
        u[r][h] = (i == 0) ? acc : rotr32(acc, 2 * i);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t b0 = (s == 0) ? B[nt][0].x : (s == 1) ? B[nt][0].z : (s == 2) ? B[nt][1].x : B[nt][1].z;
      const uint32_t b1 = (s == 0) ? B[nt][0].y : (s == 1) ? B[nt][0].w : (s == 2) ? B[nt][1].y : B[nt][1].w;
      mma_u8s8(C[nt], u[0][0], u[1][0], u[0][1], u[1][1], b0, b1);
    }
  }
}

template <int K0, int NP, int NT>
__device__ __forceinline__ void tile_compute(const uint8_t* stage, int tg, int gl_begin, int slice_goff,
                                             const int8_t* digits, int digit_stride, int ndrows,
                                             const float* inv_scale, const int32_t* gsum, int ngroups_slice,
                                             int two_c, int mt, int lane, float (&acc)[NT][2]) {
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * mt + g;
  const uint8_t* planes = stage + 256 * tg;
  for (int gl = gl_begin; gl < tg; gl += 2) {
    const int gs = slice_goff + gl;  // group index within the slice
    uint4 B[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int row = 8 * nt + g;
      if (row < ndrows) {
        const uint4* src = reinterpret_cast<const uint4*>(digits + (size_t)row * digit_stride + 128 * gs + 32 * t);
        B[nt][0] = src[0];
        B[nt][1] = src[1];
      } else {
        B[nt][0] = make_uint4(0, 0, 0, 0);
        B[nt][1] = make_uint4(0, 0, 0, 0);
      }
    }
    uint2 W[4][2];
#pragma unroll
    for (int kk = 0; kk < NP; ++kk) {
      const uint8_t* pk = planes + 2048 * (kk * tg + gl);
      W[kk][0] = *reinterpret_cast<const uint2*>(pk + 32 * r0 + 8 * t);
      W[kk][1] = *reinterpret_cast<const uint2*>(pk + 32 * (r0 + 8) + 8 * t);
    }
    int32_t C[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) C[nt][0] = C[nt][1] = C[nt][2] = C[nt][3] = 0;
    group_mma<K0, NP, NT>(W, B, C);
    const float* sc = reinterpret_cast<const float*>(stage + 256 * gl);
    const float s0 = sc[r0], s1 = sc[r0 + 8];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int bb = 4 * nt + t;  // batch row held by this lane
      const int32_t X = gsum[bb * ngroups_slice + gs];
      const float h = 0.5f * inv_scale[bb * ngroups_slice + gs];
      const int32_t v0 = C[nt][0] * 512 + C[nt][1] * 2 + two_c * X;
      const int32_t v1 = C[nt][2] * 512 + C[nt][3] * 2 + two_c * X;
      acc[nt][0] = fmaf(static_cast<float>(v0), s0 * h, acc[nt][0]);
      acc[nt][1] = fmaf(static_cast<float>(v1), s1 * h, acc[nt][1]);
    }
  }
}

template <int NT>
__device__ __forceinline__ void dispatch_tile(int k0, int np, const uint8_t* stage, int tg, int gl_begin,
                                              int slice_goff, const int8_t* digits, int digit_stride, int ndrows,
                                              const float* inv_scale, const int32_t* gsum, int ngs, int two_c,
                                              int mt, int lane, float (&acc)[NT][2]) {
#define FL_TILE(K0_, NP_)                                                                                        \
  tile_compute<K0_, NP_, NT>(stage, tg, gl_begin, slice_goff, digits, digit_stride, ndrows, inv_scale, gsum, ngs, \
                             two_c, mt, lane, acc)
  switch (k0 * 8 + np) {
    case 0 * 8 + 1: FL_TILE(0, 1); break;
    case 0 * 8 + 2: FL_TILE(0, 2); break;
    case 0 * 8 + 3: FL_TILE(0, 3); break;
    case 0 * 8 + 4: FL_TILE(0, 4); break;
    case 1 * 8 + 1: FL_TILE(1, 1); break;
    case 1 * 8 + 2: FL_TILE(1, 2); break;
    case 1 * 8 + 3: FL_TILE(1, 3); break;
    case 2 * 8 + 1: FL_TILE(2, 1); break;
    case 2 * 8 + 2: FL_TILE(2, 2); break;
    case 3 * 8 + 1: FL_TILE(3, 1); break;
    default: break;
  }
#undef FL_TILE
}

// 2 (c_b - c_a) with c_0 = 128: the constant part of the read, doubled so it is an integer.
__device__ __forceinline__ int two_c_of(int k0, int np) {
  const int b = 2 * (k0 + np), a = 2 * k0;
  const int cb2 = (1 << (8 - b)) - 1;
  const int ca2 = (a == 0) ? 256 : (1 << (8 - a)) - 1;
  return cb2 - ca2;
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int MAXP, int NT>
__global__ void __launch_bounds__(kThreads, 1) plane_gemv_kernel(const __grid_constant__ Args<MAXP> a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ float xfer[4][NT][2][32];  // gp = 1 warps hand their sums to gp = 0
  __shared__ int s_ticket;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u_begin = a.cta_begin[blockIdx.x], u_end = a.cta_begin[blockIdx.x + 1];
  if (u_begin >= u_end) return;

  uint8_t* stages = smem;
  int8_t* digits = reinterpret_cast<int8_t*>(smem + kStages * kStageBytes);
  const int ndrows = 2 * a.batch;
  float* inv_scale = reinterpret_cast<float*>(smem + kStages * kStageBytes + (size_t)ndrows * a.digit_stride);
  int32_t* gsum = reinterpret_cast<int32_t*>(inv_scale + 4 * NT * a.max_slice_groups);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      UnitCursor c = cursor_at(a, u_begin);
      for (; c.u < u_end; cursor_next(a, c)) {
        const Problem& P = a.p[c.p];
        int k0, np;
        plane_range(a, P, c.b, k0, np);
        if (np == 0) continue;
        const int tgm = tile_groups(np);
        const int g0s = slice_g0(P, c.j), ngs = slice_ng(P, c.j);
        const uint8_t* blk = P.store + (size_t)c.b * 8448u * P.G;
        for (int g0 = 0; g0 < ngs; g0 += tgm) {
          const int tg = min(tgm, ngs - g0);
          if (issued >= (uint32_t)kStages) {
            if (!mbar_wait(&empty_bar[s], phase ^ 1u)) {
              atomicExch(&g_error, 1);
              return;
            }
          }
          uint8_t* st = stages + s * kStageBytes;
          const uint32_t bytes = 256u * tg + 2048u * tg * np;
          mbar_expect_tx(&full_bar[s], bytes);
          const int gg = g0s + g0;
          bulk_g2s(st, blk + 256u * gg, 256u * tg, &full_bar[s]);
          for (int kk = 0; kk < np; ++kk)
            bulk_g2s(st + 256 * tg + 2048 * tg * kk, blk + 256u * P.G + 2048u * ((size_t)P.G * (k0 + kk) + gg),
                     2048u * tg, &full_bar[s]);
          ++issued;
          if (++s == kStages) {
            s = 0;
            phase ^= 1u;
          }
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int mt = warp & 3, gp = warp >> 2;
  int s = 0;
  uint32_t phase = 0;
  int cur_p = -1, cur_j = -1;
  UnitCursor c = cursor_at(a, u_begin);
  for (; c.u < u_end; cursor_next(a, c)) {
    const Problem& P = a.p[c.p];
    const int ngs = slice_ng(P, c.j);
    if (c.p != cur_p || c.j != cur_j) {
      named_bar(1, 32 * kConsumerWarps);
      XDigitView v;
      v.digits = digits;
      v.inv_scale = inv_scale;
      v.gsum = gsum;
      v.stride = a.digit_stride;
      v.ngroups = ngs;
      build_x_digits(P.x, P.G * 128, a.batch, 4 * NT, 128 * slice_g0(P, c.j), v, 1, threadIdx.x,
                     32 * kConsumerWarps);
      named_bar(1, 32 * kConsumerWarps);
      cur_p = c.p;
      cur_j = c.j;
    }
    int k0, np;
    plane_range(a, P, c.b, k0, np);
    const int row_base = 64 * c.b + 16 * mt;
    const int g = lane >> 2, t = lane & 3;
    if (np == 0) {
      if (a.mode == 0 && c.j == 0 && gp == 0) {
        for (int nt = 0; nt < NT; ++nt) {
          const int bb = 4 * nt + t;
          if (bb < a.batch) {
            P.y[(size_t)bb * 64 * P.nblocks + row_base + g] = 0.f;
            P.y[(size_t)bb * 64 * P.nblocks + row_base + g + 8] = 0.f;
          }
        }
      }
      continue;
    }
    float acc[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
    const int tgm = tile_groups(np);
    const int two_c = two_c_of(k0, np);
    for (int g0 = 0; g0 < ngs; g0 += tgm) {
      const int tg = min(tgm, ngs - g0);
      if (!mbar_wait(&full_bar[s], phase)) {
        atomicExch(&g_error, 2);
        return;
      }
      dispatch_tile<NT>(k0, np, stages + s * kStageBytes, tg, gp, g0, digits, a.digit_stride, ndrows, inv_scale,
                        gsum, ngs, two_c, mt, lane, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
      if (++s == kStages) {
        s = 0;
        phase ^= 1u;
      }
    }
    // combine the two group parities of each m-tile
    if (gp == 1) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        xfer[mt][nt][0][lane] = acc[nt][0];
        xfer[mt][nt][1][lane] = acc[nt][1];
      }
    }
    named_bar(2 + mt, 64);
    if (gp == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[nt][0] += xfer[mt][nt][0][lane];
        acc[nt][1] += xfer[mt][nt][1][lane];
      }
    }
    named_bar(2 + mt, 64);
    const size_t ystride = (size_t)64 * P.nblocks;
    if (P.slices == 1) {
      if (gp == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int bb = 4 * nt + t;
          if (bb < a.batch) {
            float* y0 = P.y + (size_t)bb * ystride + row_base + g;
            if (a.mode == 0) {
              y0[0] = acc[nt][0];
              y0[8] = acc[nt][1];
            } else {
              y0[0] += acc[nt][0];
              y0[8] += acc[nt][1];
            }
          }
        }
      }
    } else {
      // partial for this slice, then the last slice to finish reduces in slice order
      if (gp == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int bb = 4 * nt + t;
          if (bb < a.batch) {
            float* pp = P.partial + (((size_t)c.j * P.nblocks + c.b) * a.batch + bb) * 64 + 16 * mt + g;
            pp[0] = acc[nt][0];
            pp[8] = acc[nt][1];
          }
        }
      }
      __threadfence();
      named_bar(1, 32 * kConsumerWarps);
      if (threadIdx.x == 0) s_ticket = (int)atomicAdd(&P.tickets[c.b], 1u);
      named_bar(1, 32 * kConsumerWarps);
      if (s_ticket == P.slices - 1) {
        __threadfence();
        for (int e = threadIdx.x; e < a.batch * 64; e += 32 * kConsumerWarps) {
          const int bb = e / 64, r = e % 64;
          float sum = 0.f;
          for (int jj = 0; jj < P.slices; ++jj)
            sum += __ldcg(P.partial + (((size_t)jj * P.nblocks + c.b) * a.batch + bb) * 64 + r);
          float* yy = P.y + (size_t)bb * ystride + 64 * c.b + r;
          if (a.mode == 0)
            *yy = sum;
          else
            *yy += sum;
        }
        if (threadIdx.x == 0) P.tickets[c.b] = 0u;
      }
    }
  }
}

// ---------------------------------------------------------------- host side

struct Plan {
  int slices, slice_groups;
};

static int digit_stride_for(int slice_groups) { return 128 * slice_groups + 16; }

// Dynamic shared memory: stages, activation digits (2 rows per batch entry),
// and per (padded batch, group) the inverse scale and the group sum.
static size_t smem_bytes(int batch, int slice_groups) {
  const int nt = (batch + 3) / 4;
  return (size_t)kStages * kStageBytes + (size_t)2 * batch * digit_stride_for(slice_groups) +
         (size_t)4 * nt * slice_groups * 8;
}

// Widest column slice (in 128-column groups) whose digits fit next to the stages.
static int max_groups_fit(int batch) {
  const int nt = (batch + 3) / 4;
  const long avail = (long)kSmemLimit - (long)kStages * kStageBytes - 32L * batch;
  return (int)std::max(1L, avail / (256L * batch + 32L * nt));
}

// Column split for a single layer: enough units to fill the GPU, slices of whole
// groups, and a slice narrow enough for the activation digits to fit in smem.
static Plan plan_single(int nblocks, int G, int batch, int nsm) {
  Plan pl;
  int max_sg = max_groups_fit(batch);
  int s_mem = (G + max_sg - 1) / max_sg;
  int s_fill = (2 * nsm + nblocks - 1) / nblocks;
  int s = std::max(s_mem, std::min(s_fill, std::max(1, G / 4)));
  s = std::min(s, G);
  pl.slice_groups = (G + s - 1) / s;
  pl.slices = (G + pl.slice_groups - 1) / pl.slice_groups;
  return pl;
}

static size_t workspace_for(const Plan& pl, int nblocks, int batch) {
  if (pl.slices <= 1) return 0;
  size_t tickets = ((size_t)nblocks * 4 + 255) / 256 * 256;
  return tickets + (size_t)pl.slices * nblocks * batch * 64 * 4;
}

template <int MAXP>
static void partition(Args<MAXP>& a, int nsm) {
  // cost of a unit ~ columns it reads; contiguous cost-balanced ranges per CTA
  double total = 0;
  for (int i = 0; i < a.nproblems; ++i) total += (double)a.p[i].nblocks * a.p[i].G;
  int units = a.p[a.nproblems - 1].unit_begin + a.p[a.nproblems - 1].nblocks * a.p[a.nproblems - 1].slices;
  int ncta = std::min(nsm, units);
  ncta = std::max(1, std::min(ncta, kMaxCtas));
  a.ncta = ncta;
  int c = 0;
  a.cta_begin[0] = 0;
  double acc = 0;
  for (int i = 0; i < a.nproblems && c < ncta; ++i) {
    const Problem& P = a.p[i];
    const int nu = P.nblocks * P.slices;
    const double per = (double)P.G / P.slices;
    for (int k = 0; k < nu; ++k) {
      acc += per;
      const int u = P.unit_begin + k + 1;
      while (c + 1 < ncta && acc >= total * (c + 1) / ncta) a.cta_begin[++c] = u;
    }
  }
  while (c + 1 < ncta) a.cta_begin[++c] = units;
  a.cta_begin[ncta] = units;
}

template <int MAXP, int NT>
static fl_status launch(const Args<MAXP>& a, cudaStream_t st) {
  const size_t smem = smem_bytes(a.batch, a.max_slice_groups);
  auto kern = plane_gemv_kernel<MAXP, NT>;
  FL_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                "cudaFuncSetAttribute(plane_gemv)");
  kern<<<a.ncta, kThreads, smem, st>>>(a);
  FL_CHECK_CUDA(cudaGetLastError(), "launch plane_gemv");
  return FL_OK;
}

template <int MAXP>
static fl_status launch_nt(const Args<MAXP>& a, cudaStream_t st) {
  switch ((a.batch + 3) / 4) {
    case 1: return launch<MAXP, 1>(a, st);
    case 2: return launch<MAXP, 2>(a, st);
    case 3: return launch<MAXP, 3>(a, st);
    default: return launch<MAXP, 4>(a, st);
  }
}

static fl_status check_weight(const fl_plane_weight* w, const char* what) {
  if (!w) return fail(FL_ERR_ARG, "%s: weight descriptor is NULL", what);
  if (!w->store) return fail(FL_ERR_ARG, "%s: plane store pointer is NULL", what);
  if (w->out <= 0 || w->in <= 0 || w->out % 64 || w->in % 128)
    return fail(FL_ERR_SHAPE, "%s: out=%d in=%d (need out %% 64 == 0, in %% 128 == 0)", what, w->out, w->in);
  if (!aligned16(w->store)) return fail(FL_ERR_ALIGN, "%s: plane store not 16-byte aligned", what);
  return FL_OK;
}

static fl_status single(const fl_plane_weight* w, const uint8_t* lv_from, const uint8_t* lv_to, const uint16_t* x,
                        int batch, float* y, void* ws, size_t ws_bytes, void* stream, int mode,
                        const char* what) {
  fl_status st = check_weight(w, what);
  if (st != FL_OK) return st;
  if (!lv_from || !x || !y || (mode == 1 && !lv_to)) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  if (!aligned16(x)) return fail(FL_ERR_ALIGN, "%s: x not 16-byte aligned", what);
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  const int nblocks = w->out / 64, G = w->in / 128;
  Plan pl = plan_single(nblocks, G, batch, nsm);
  const size_t need = workspace_for(pl, nblocks, batch);
  if (need > 0 && (!ws || ws_bytes < need))
    return fail(FL_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", what, ws ? ws_bytes : (size_t)0, need);
  if (need > 0 && !aligned16(ws)) return fail(FL_ERR_ALIGN, "%s: workspace not 16-byte aligned", what);
  static thread_local Args<1> a;
  a.nproblems = 1;
  a.batch = batch;
  a.mode = mode;
  a.max_slice_groups = pl.slice_groups;
  a.digit_stride = digit_stride_for(pl.slice_groups);
  Problem& P = a.p[0];
  P.store = w->store;
  P.lv_from = lv_from;
  P.lv_to = lv_to;
  P.x = x;
  P.y = y;
  P.nblocks = nblocks;
  P.G = G;
  P.slices = pl.slices;
  P.slice_groups = pl.slice_groups;
  P.unit_begin = 0;
  if (pl.slices > 1) {
    size_t tick = ((size_t)nblocks * 4 + 255) / 256 * 256;
    P.tickets = reinterpret_cast<uint32_t*>(ws);
    P.partial = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + tick);
  } else {
    P.tickets = nullptr;
    P.partial = nullptr;
  }
  partition(a, nsm);
  return launch_nt(a, static_cast<cudaStream_t>(stream));
}

}  // namespace gemv
}  // namespace fl

using namespace fl;

extern "C" size_t fl_gemv_workspace_bytes(int out, int in, int batch) {
  if (out <= 0 || in <= 0 || out % 64 || in % 128 || batch < 1 || batch > FL_MAX_BATCH) return 0;
  const int nsm = device_sm_count();
  if (nsm <= 0) return 0;
  gemv::Plan pl = gemv::plan_single(out / 64, in / 128, batch, nsm);
  return gemv::workspace_for(pl, out / 64, batch);
}

extern "C" fl_status fl_gemv_depth(const fl_plane_weight* w, const uint8_t* levels, const uint16_t* x, int batch,
                                   float* y, void* workspace, size_t workspace_bytes, void* stream) {
  return gemv::single(w, levels, nullptr, x, batch, y, workspace, workspace_bytes, stream, 0, "fl_gemv_depth");
}

extern "C" fl_status fl_gemv_residual(const fl_plane_weight* w, const uint8_t* from_levels,
                                      const uint8_t* to_levels, const uint16_t* x, int batch, float* y,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  return gemv::single(w, from_levels, to_levels, x, batch, y, workspace, workspace_bytes, stream, 1,
                      "fl_gemv_residual");
}

extern "C" fl_status fl_gemv_batched(const fl_gemv_problem* problems, int n, int batch, int mode, void* stream) {
  const char* what = "fl_gemv_batched";
  if (!problems) return fail(FL_ERR_ARG, "%s: problems is NULL", what);
  if (n < 1 || n > FL_MAX_PROBLEMS) return fail(FL_ERR_ARG, "%s: n=%d (1..%d)", what, n, FL_MAX_PROBLEMS);
  if (mode != 0 && mode != 1) return fail(FL_ERR_ARG, "%s: mode=%d (0 depth, 1 residual)", what, mode);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  static thread_local gemv::Args<FL_MAX_PROBLEMS> a;
  a.nproblems = n;
  a.batch = batch;
  a.mode = mode;
  int max_g = 0, unit = 0;
  for (int i = 0; i < n; ++i) {
    const fl_gemv_problem& q = problems[i];
    fl_status st = gemv::check_weight(&q.w, what);
    if (st != FL_OK) return st;
    if (!q.levels || !q.x || !q.y || (mode == 1 && !q.to_levels))
      return fail(FL_ERR_ARG, "%s: problem %d has a NULL pointer", what, i);
    if (!aligned16(q.x)) return fail(FL_ERR_ALIGN, "%s: problem %d x not 16-byte aligned", what, i);
    const int G = q.w.in / 128;
    if (G > gemv::max_groups_fit(batch))
      return fail(FL_ERR_SHAPE, "%s: problem %d in=%d too wide for batch %d in one launch (in <= %d)", what, i,
                  q.w.in, batch, 128 * gemv::max_groups_fit(batch));
    gemv::Problem& P = a.p[i];
    P.store = q.w.store;
    P.lv_from = q.levels;
    P.lv_to = q.to_levels;
    P.x = q.x;
    P.y = q.y;
    P.partial = nullptr;
    P.tickets = nullptr;
    P.nblocks = q.w.out / 64;
    P.G = G;
    P.slices = 1;
    P.slice_groups = G;
    P.unit_begin = unit;
    unit += P.nblocks;
    max_g = std::max(max_g, G);
  }
  a.max_slice_groups = max_g;
  a.digit_stride = gemv::digit_stride_for(max_g);
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  gemv::partition(a, nsm);
  return gemv::launch_nt(a, static_cast<cudaStream_t>(stream));
}
