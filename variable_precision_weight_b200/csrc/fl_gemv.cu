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
//  * Work unit = (problem, column slice, 64-row block); each CTA owns a
//    contiguous, cost-balanced range of units.
//  * Four consumer teams of four warps. A team owns whole units (its four
//    warps are the block's four 16-row m-tiles, so a warp's row sums are
//    final when the unit ends) and two private stages of the shared-memory
//    ring. Units go to the teams round-robin.
//  * A producer warp caches the levels of the CTA's units in shared memory,
//    then walks the four teams' unit streams, claims a team's next free
//    stage, writes a tile header and issues 1-D bulk copies of the scales and
//    of the planes the block's depth needs (one copy when the tile spans the
//    whole row). Planes the depth does not need are never fetched.
//  * Per 128-column group a warp assembles the code bytes u_d of its rows
//    from the plane words with one AND/OR per plane and one rotate per four
//    columns (the store layout places each plane's field so that this yields
//    u_d in byte lanes), feeds them as the u8 operand of mma.sync m16n8k32
//    against the activations written as four signed int8 digits of a 31-bit
//    per-group fixed point (built once per CTA for every slice it touches;
//    the digits go in as two pairs per batch row, each pair an MMA column
//    pair), and turns the int32 group sums into fp32 with the group scale
//    and the constant part (c_b - c_a) sum_c x_c; the two pairs' sums meet
//    in one shuffle when the unit ends.
//  * Layers with too few blocks to fill the GPU are split into column slices;
//    a slice writes a partial to the caller's workspace and the last team to
//    finish a block (atomic ticket) adds the slices in order. No CTA ever
//    waits on another; every mbarrier wait is bounded.
#include <algorithm>
#include <mutex>
#include <vector>

#include "fl_common.cuh"
#include "fl_gate_merge.cuh"

namespace fl {

// The tensor-core (tcgen05) path of fl_gemv_tc.cu: single-layer calls at batches from 9 up to
// FL_MAX_GEMV_BATCH.
bool tc_takes(int batch);
size_t tc_workspace_bytes(int out, int in, int batch);
fl_status tc_single(const fl_plane_weight* w, const uint8_t* lv_from, const uint8_t* lv_to, const uint16_t* x,
                    int batch, float* y, void* ws, size_t ws_bytes, void* stream, int mode, const char* what);

namespace gemv {

constexpr int kTeams = 4;
constexpr int kTeamWarps = 4;
constexpr int kTeamThreads = 32 * kTeamWarps;
constexpr int kConsumerWarps = kTeams * kTeamWarps;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kProducerWarps = kTeams;  // producer warp t feeds team t
constexpr int kThreads = kConsumers + 32 * kProducerWarps;
constexpr int kTeamStages = 2;
constexpr int kStages = kTeams * kTeamStages;
constexpr int kMaxCtas = 960;   // unit ranges per launch (bounded by the kernel-parameter space)
constexpr int kRed = 8;               // outputs per thread per pass of the slice reduction
constexpr int kMaxSlots = 64;         // distinct (problem, slice) pairs one CTA may touch
constexpr int kLevelCache = 4096;     // most units per CTA; all their plane ranges are cached in smem
constexpr int kListCache = 512;       // most units per CTA of a listed pass; their block indices are cached
constexpr int kSkipUnit = 0xFF;       // level-cache mark of a listed unit whose block index is out of range
constexpr int kSmemLimit = 232448 - 16384;  // opt-in shared memory per block on B200, less static use
// Stage size by N-tile count: 18 KB tiles while the products are light (batch <= 4); half that
// at larger batches, whose four-digit activations need the shared memory and whose math per
// weight byte is several times heavier, so fewer bytes in flight still keep up.
__host__ __device__ constexpr int stage_bytes(int nt) { return nt <= 2 ? 18432 : 9216; }
__host__ __device__ constexpr int digit_budget(int nt) { return kSmemLimit - kStages * stage_bytes(nt); }

// Groups per tile for np planes: largest tg with tg * (256 + 2048 np) <= stage_bytes(nt)
// (8, 4, 2, 2 groups for 1-4 planes at 18 KB; 4, 2, 1, 1 at 9 KB).
__host__ __device__ constexpr int tile_groups(int np, int nt) { return stage_bytes(nt) / (256 + 2048 * np); }

struct Problem {
  const uint8_t* store;
  const uint8_t* lv_from;
  const uint8_t* lv_to;
  const uint16_t* x;
  float* y;
  float* partial;      // [slices][nblocks][batch][64] when slices > 1
  uint32_t* tickets;   // [nblocks] when slices > 1
  int nblocks;          // units per slice: the layer's blocks, or the listed ones
  int G;
  int slices;
  int slice_groups;    // groups per slice (last slice shorter)
  int unit_begin;      // first global unit index of this problem
  const int32_t* list; // listed pass: unit i is block list[i] (NULL: unit i is block i)
  int ynb;             // blocks of the layer (its output rows / 64)
};

template <int MAXP>
struct Args {
  int nproblems;
  int batch;
  int mode;            // 0 depth (y =), 1 residual (y +=)
  int ncta;
  int cta_begin[kMaxCtas + 1];
  int cta_slice[kMaxCtas];  // first (problem, slice) pair of the CTA, counted in order, << 7 | pairs touched
  // fused logit gate over problem gate_p's outputs (gate_p < 0: none)
  int gate_p;
  float tau_h, tau_m;
  float* entropy;
  float* margin;
  int32_t* top2;
  uint8_t* escalate;
  uint32_t* gate_ticket;   // launch counter, zero between launches
  GateRec* gate_part;      // [kMaxCtas][FL_MAX_BATCH] per-CTA partials
  int gate_cta0, gate_ncta;  // the CTAs whose unit ranges hold gate-problem units
  // conditional launch: the pass runs only if *run_if != 0 (run_if NULL: always); runs
  // (optional) counts the passes that ran
  const uint8_t* run_if;
  uint32_t* runs;
  // the fused gate's merged record per batch row is written here instead of the gate's outputs
  // (a rank's piece of a vocabulary split over devices), indices offset by gate_index_base
  GateRec* gate_partial;
  int gate_index_base;
  int listed;          // some problem has a block list (units per CTA <= kListCache)
  Problem p[MAXP];
};

__device__ int g_error;  // set when a bounded wait runs out (never expected)

// One (problem, column slice) touched by a CTA: the units [u0, u1) of the CTA's range (relative
// to its first unit) are its blocks b0, b0 + 1, ...; everything the producer and consumers need
// is copied here once, so the hot loops never index the kernel-parameter problem table.
// Activation digits (fl_common.cuh): rows 4b .. 4b+3 hold digits d3, d2, d1, d0 of batch row b
// (stride bytes per row), i.e. digit pair p = 2b + r (r = 0: d3 d2, r = 1: d1 d0) is rows 2p,
// 2p+1; gconst[(padded pair row) * ngroups + group] = (pair weight, constant part): (2^(16 -
// sigma), 2^-sigma sum_c v_c) for r = 0 and (2^-sigma, 0) for r = 1.
struct __align__(16) Slot {
  int p, j, u0, u1, b0;
  int nblocks, G, ngroups, slices, gfirst;  // gfirst = first group of the slice in the row
  int ynb;           // blocks of the layer's output (rows / 64)
  int stride;
  int it0;           // first (batch row, group) digit item of the slot in the CTA's item count
  uint32_t digits;   // smem address
  uint32_t gconst;   // smem address
  const uint8_t* store;
  const uint8_t* lv_from;
  const uint8_t* lv_to;
  const uint16_t* x;
  float* y;
  float* partial;
  uint32_t* tickets;
  const int32_t* list;  // listed pass: the slot's units are blocks list[b0 ..]
};

__device__ __forceinline__ int slice_ng(const Problem& P, int j) {
  return min(P.slice_groups, P.G - j * P.slice_groups);
}

// Mask selecting plane k's fields for column set i (rotl(0x03030303, 6-2k+2i)).
__host__ __device__ constexpr uint32_t plane_mask(int k, int i) {
  return (((6 - 2 * k + 2 * i) & 7) == 0)
             ? 0x03030303u
             : ((0x03030303u << ((6 - 2 * k + 2 * i) & 7)) | (0x03030303u >> (32 - ((6 - 2 * k + 2 * i) & 7))));
}

// Named barriers: 0 is __syncthreads; team t uses kBarTeam0 + t.
enum : int { kBarGate = 1, kBarTeam0 = 2, kBarProducers = 6, kBarLevels = 7, kBarX = 8 };

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// c_b - c_a with c_0 = 128: the constant part of the read of planes [k0, k0 + np).
__device__ __forceinline__ float cfac_of(int k0, int np) {
  const int b = 2 * (k0 + np), a = 2 * k0;
  const int cb2 = (1 << (8 - b)) - 1;
  const int ca2 = (a == 0) ? 256 : (1 << (8 - a)) - 1;
  return 0.5f * (float)(cb2 - ca2);
}

// Digit items of every slot (one item = 128 columns of one batch row) by nthreads consumer
// threads, tid in [0, nthreads): one warp per item, four items' loads in flight per warp.
// See fl_common.cuh for the number format.
__device__ __forceinline__ void convert_item(uint2 raw, const Slot& sl, int b, int g, int lane) {
  const float f[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
  uint32_t dw[4];
  int2 part;
  const int sigma = split_digits(f, dw, part);
  const uint32_t dh = sl.digits + (uint32_t)((4 * b) * sl.stride + 128 * g + 4 * lane);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(dh + (uint32_t)(k * sl.stride)), "r"(dw[k]) : "memory");
  part.x = __reduce_add_sync(0xffffffffu, part.x);
  part.y = __reduce_add_sync(0xffffffffu, part.y);
  if (lane == 0) {
    const uint32_t gc = sl.gconst + 8u * (uint32_t)(2 * b * sl.ngroups + g);
    asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(gc), "f"(ldexpf(1.0f, 16 - sigma)),
                 "f"(ldexpf(fmaf(65536.f, (float)part.x, (float)part.y), -sigma))
                 : "memory");
    asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(gc + 8u * (uint32_t)sl.ngroups), "f"(ldexpf(1.0f, -sigma)),
                 "f"(0.f)
                 : "memory");
  }
}

// When the items take more than one round (`multi`, large batches), every warp arrives on kBarX
// once its last round's loads are issued, and the producers hold the weight stream until then,
// so no activation read queues behind it.
__device__ __forceinline__ void build_digits(const Slot* slots, int nsl, int batch, int batch_pad, int tid,
                                             int nthreads, int total, bool multi) {
  const int lane = tid & 31, wid = tid >> 5, nw = nthreads >> 5;
  int si = 0;
  if (multi && wid >= total) bar_arrive(kBarX, kThreads);
  for (int it0 = wid; it0 < total; it0 += 4 * nw) {
    uint2 raw[4];
    int sq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int it = it0 + q * nw;
      sq[q] = -1;
      if (it < total) {
        while (si + 1 < nsl && it >= slots[si + 1].it0) ++si;
        const Slot& sl = slots[si];
        const int local = it - sl.it0, b = local / sl.ngroups, g = local % sl.ngroups;
        raw[q] = __ldg(reinterpret_cast<const uint2*>(sl.x + (size_t)b * sl.G * 128 + 128 * (sl.gfirst + g) +
                                                      4 * lane));
        sq[q] = si;
      }
    }
    if (multi && it0 + 4 * nw >= total) bar_arrive(kBarX, kThreads);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (sq[q] >= 0) {
        const Slot& sl = slots[sq[q]];
        const int local = it0 + q * nw - sl.it0;
        convert_item(raw[q], sl, local / sl.ngroups, local % sl.ngroups, lane);
      }
    }
  }
  // padded pair rows read zero constants
  for (int i = 0; i < nsl; ++i) {
    const Slot& sl = slots[i];
    for (int e = tid; e < (batch_pad - 2 * batch) * sl.ngroups; e += nthreads)
      asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(sl.gconst + 8u * (uint32_t)(2 * batch * sl.ngroups + e)),
                   "f"(0.f), "f"(0.f)
                   : "memory");
  }
}

// Large batches: the activation rows of every slot arrive by one 1-D bulk copy per (slot, batch
// row) into the idle stage buffers (item `it` at smem offset 256 it, x_bar tracks the bytes), so
// they all take one round trip; the consumers then convert from shared memory.
__device__ __forceinline__ void stage_x(const Slot* slots, int nsl, int batch, uint8_t* smem, uint64_t* x_bar,
                                        int ditems) {
  mbar_expect_tx(x_bar, (uint32_t)ditems * 256u);
  for (int i = 0; i < nsl; ++i) {
    const Slot& sl = slots[i];
    for (int b = 0; b < batch; ++b)
      bulk_g2s(smem + (size_t)(sl.it0 + b * sl.ngroups) * 256u,
               sl.x + (size_t)b * sl.G * 128 + 128 * sl.gfirst, 256u * sl.ngroups, x_bar);
  }
}

__device__ __forceinline__ void convert_staged(const Slot* slots, int nsl, int batch, int batch_pad,
                                               const uint8_t* smem, int tid, int nthreads, int total) {
  const int lane = tid & 31, wid = tid >> 5, nw = nthreads >> 5;
  const uint32_t base = smem_u32(smem);
  int si = 0;
  for (int it = wid; it < total; it += nw) {
    while (si + 1 < nsl && it >= slots[si + 1].it0) ++si;
    const Slot& sl = slots[si];
    const int local = it - sl.it0;
    uint2 raw;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(raw.x), "=r"(raw.y) : "r"(base + 256u * it + 8u * lane));
    convert_item(raw, sl, local / sl.ngroups, local % sl.ngroups, lane);
  }
  for (int i = 0; i < nsl; ++i) {
    const Slot& sl = slots[i];
    for (int e = tid; e < (batch_pad - 2 * batch) * sl.ngroups; e += nthreads)
      asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(sl.gconst + 8u * (uint32_t)(2 * batch * sl.ngroups + e)),
                   "f"(0.f), "f"(0.f)
                   : "memory");
  }
}

// One group (128 columns) of a tile for one warp (rows r0 and r0 + 8): plane words, code bytes
// by mask / or / rotate, 4 k32 MMAs per N-tile, then the group's scale and constant part.
template <int K0, int NP, int NT>
__device__ __forceinline__ void group_compute(uint32_t wrow, uint32_t srow, int tg, int gl, const uint32_t (&dlane)[NT],
                                              const uint32_t (&dstep)[NT], uint32_t gc_lane, int gstride,
                                              int slice_goff, float cfac, int t, float (&acc)[NT][2]) {
      const int gs = slice_goff + gl;
      uint2 W[NP][2];
#pragma unroll
      for (int kk = 0; kk < NP; ++kk) {
        const uint32_t pk = wrow + 2048u * (kk * tg + gl);
        W[kk][0] = lds_v2(pk);
        W[kk][1] = lds_v2(pk + 256u);
      }
      const float s0 = lds_f32(srow + 256u * gl), s1 = lds_f32(srow + 256u * gl + 32u);
      if constexpr (NT > 1) {
        // Several N-tiles: build the group's four k-step A operands once, then one N-tile at a
        // time (its fragment, four MMAs, its fold), which keeps the live registers per N-tile.
        uint32_t u4[4][2][2];
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          const int w = st >> 1;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int i = 2 * (st & 1) + h;
              uint32_t v = 0;
#pragma unroll
              for (int kk = 0; kk < NP; ++kk) v |= (w ? W[kk][r].y : W[kk][r].x) & plane_mask(K0 + kk, i);
              u4[st][r][h] = (i == 0) ? v : rotr32(v, 2 * i);
            }
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t src = dlane[nt] + dstep[nt] * (uint32_t)gs;
          const uint4 B0 = lds_v4(src), B1 = lds_v4(src + 16u);
          int32_t C[4] = {0, 0, 0, 0}, D[4] = {0, 0, 0, 0};
          mma_u8s8(C, u4[0][0][0], u4[0][1][0], u4[0][0][1], u4[0][1][1], B0.x, B0.y);
          mma_u8s8(C, u4[1][0][0], u4[1][1][0], u4[1][0][1], u4[1][1][1], B0.z, B0.w);
          mma_u8s8(D, u4[2][0][0], u4[2][1][0], u4[2][0][1], u4[2][1][1], B1.x, B1.y);
          mma_u8s8(D, u4[3][0][0], u4[3][1][0], u4[3][0][1], u4[3][1][1], B1.z, B1.w);
          const float2 hc = lds_f2(gc_lane + 8u * (uint32_t)(nt * 4 * gstride + gs));
          const float off = cfac * hc.y;
          const float v0 = fmaf((float)((C[0] + D[0]) * 256 + (C[1] + D[1])), hc.x, off);
          const float v1 = fmaf((float)((C[2] + D[2]) * 256 + (C[3] + D[3])), hc.x, off);
          acc[nt][0] = fmaf(v0, s0, acc[nt][0]);
          acc[nt][1] = fmaf(v1, s1, acc[nt][1]);
        }
      } else {
      uint4 B[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t src = dlane[nt] + dstep[nt] * (uint32_t)gs;
        B[nt][0] = lds_v4(src);
        B[nt][1] = lds_v4(src + 16u);
      }
      int32_t C[NT][4], D[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        C[nt][0] = C[nt][1] = C[nt][2] = C[nt][3] = 0;
        D[nt][0] = D[nt][1] = D[nt][2] = D[nt][3] = 0;
      }
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        const int w = st >> 1;
        const int i0 = 2 * (st & 1), i1 = i0 + 1;
        uint32_t u[2][2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int i = h ? i1 : i0;
            uint32_t v = 0;
#pragma unroll
            for (int kk = 0; kk < NP; ++kk) v |= (w ? W[kk][r].y : W[kk][r].x) & plane_mask(K0 + kk, i);
            u[r][h] = (i == 0) ? v : rotr32(v, 2 * i);
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t b0 = (st == 0) ? B[nt][0].x : (st == 1) ? B[nt][0].z : (st == 2) ? B[nt][1].x : B[nt][1].z;
          const uint32_t b1 = (st == 0) ? B[nt][0].y : (st == 1) ? B[nt][0].w : (st == 2) ? B[nt][1].y : B[nt][1].w;
          if (st < 2)
            mma_u8s8(C[nt], u[0][0], u[1][0], u[0][1], u[1][1], b0, b1);
          else
            mma_u8s8(D[nt], u[0][0], u[1][0], u[0][1], u[1][1], b0, b1);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float2 hc = lds_f2(gc_lane + 8u * (uint32_t)(nt * 4 * gstride + gs));
        const float off = cfac * hc.y;
        const float v0 = fmaf((float)((C[nt][0] + D[nt][0]) * 256 + (C[nt][1] + D[nt][1])), hc.x, off);
        const float v1 = fmaf((float)((C[nt][2] + D[nt][2]) * 256 + (C[nt][3] + D[nt][3])), hc.x, off);
        acc[nt][0] = fmaf(v0, s0, acc[nt][0]);
        acc[nt][1] = fmaf(v1, s1, acc[nt][1]);
      }
      }
}

// One tile for one warp: all tg groups of the tile. At batch <= 4 a full tile runs with a
// compile-time group count, so the groups' loads and MMAs interleave freely; with more
// N-tiles the groups run one after the other, which keeps the registers in bounds.
template <int K0, int NP, int NT, bool FULL>
__device__ __forceinline__ void tile_compute(uint32_t stage, int tg_arg, const uint32_t (&dlane)[NT],
                                             const uint32_t (&dstep)[NT], uint32_t gc_lane, int gstride,
                                             int slice_goff, float cfac, int r0, int t, float (&acc)[NT][2]) {
  constexpr int TG = tile_groups(NP, NT);
  const int tg = FULL ? TG : tg_arg;
  const uint32_t planes = stage + 256u * tg;
  const uint32_t wrow = planes + 32u * r0 + 8u * t;
  const uint32_t srow = stage + 4u * r0;
  if constexpr (NT == 1) {
#pragma unroll
    for (int gl = 0; gl < TG; ++gl)
      if (FULL || gl < tg)
        group_compute<K0, NP, NT>(wrow, srow, tg, gl, dlane, dstep, gc_lane, gstride, slice_goff, cfac, t, acc);
  } else {
#pragma unroll 1
    for (int gl = 0; gl < tg; ++gl)
      group_compute<K0, NP, NT>(wrow, srow, tg, gl, dlane, dstep, gc_lane, gstride, slice_goff, cfac, t, acc);
  }
}

template <int NT>
__device__ __forceinline__ void dispatch_tile(int k0, int np, uint32_t stage, int tg, const uint32_t (&dlane)[NT],
                                              const uint32_t (&dstep)[NT], uint32_t gc_lane, int gstride,
                                              int slice_goff, float cfac, int r0, int t, float (&acc)[NT][2]) {
#define FL_TILE(K0_, NP_)                                                                            \
  if (NT == 1 && tg == tile_groups(NP_, NT))                                                            \
    tile_compute<K0_, NP_, NT, true>(stage, tg, dlane, dstep, gc_lane, gstride, slice_goff, cfac, r0, t, acc); \
  else                                                                                               \
    tile_compute<K0_, NP_, NT, false>(stage, tg, dlane, dstep, gc_lane, gstride, slice_goff, cfac, r0, t, acc)
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

// ---------------------------------------------------------------- fused logit gate
// Per consumer warp and batch row, a running partial (in dynamic shared memory at gw) over
// the gate problem's outputs this warp produced; merged per CTA by the last warp to finish,
// per launch by the last CTA to finish (atomic counters, no waiting).

__device__ __forceinline__ GateRec ldcg_rec(const GateRec* p) {
  const float4 u = __ldcg(reinterpret_cast<const float4*>(p));
  const int4 w = __ldcg(reinterpret_cast<const int4*>(p) + 1);
  GateRec r;
  r.m = u.x;
  r.S = u.y;
  r.T = u.z;
  r.v2 = u.w;
  r.i1 = w.x;
  r.i2 = w.y;
  r.pad0 = r.pad1 = 0;
  return r;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Warp 0 publishes the CTA's partials (lane bb holds batch row bb's): lane 0 stores them and
// takes the launch counter with one acquire-release atomic; the last CTA merges every CTA's
// partials in CTA order and writes the gate outputs.
template <int MAXP>
__device__ __forceinline__ void gate_publish(const Args<MAXP>& a, const GateRec& mine, int lane) {
  GateRec* part = a.gate_part + (size_t)(blockIdx.x - a.gate_cta0) * FL_MAX_BATCH;
  int last = 0;
  for (int bb = 0; bb < a.batch; ++bb) {
    GateRec r;
    r.m = __shfl_sync(0xffffffffu, mine.m, bb);
    r.S = __shfl_sync(0xffffffffu, mine.S, bb);
    r.T = __shfl_sync(0xffffffffu, mine.T, bb);
    r.v2 = __shfl_sync(0xffffffffu, mine.v2, bb);
    r.i1 = __shfl_sync(0xffffffffu, mine.i1, bb);
    r.i2 = __shfl_sync(0xffffffffu, mine.i2, bb);
    r.pad0 = r.pad1 = 0;
    if (lane == 0) part[bb] = r;
  }
  if (lane == 0) last = (atom_add_acq_rel(a.gate_ticket, 1u) == (uint32_t)(a.gate_ncta - 1));
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  for (int bb = 0; bb < a.batch; ++bb) {
    // lane 0 acquired the counter; the others' loads are ordered after it by the warp sync
    __syncwarp();
    GateRec r = empty_rec();
    for (int c = lane; c < a.gate_ncta; c += 32) r = merge2(r, ldcg_rec(&a.gate_part[(size_t)c * FL_MAX_BATCH + bb]));
    r = warp_merge(r);
    if (lane == 0) {
      if (a.gate_partial) {
        if (r.i1 != 0x7fffffff) r.i1 += a.gate_index_base;  // no index (an empty piece) stays so
        if (r.i2 != 0x7fffffff) r.i2 += a.gate_index_base;
        a.gate_partial[bb] = r;
      } else {
        gate_outputs(r, a.tau_h, a.tau_m, a.entropy + bb, a.margin + bb, a.top2 + 2 * bb, a.escalate + bb);
      }
    }
  }
  if (lane == 0) *a.gate_ticket = 0u;
}

// The consumer warps' partials gws [kConsumerWarps][batch] are in shared memory: warp 0 merges
// them (one lane per warp) and publishes.
template <int MAXP>
__device__ __forceinline__ void gate_cta_finish(const Args<MAXP>& a, const GateRec* gws, int warp, int lane) {
  named_bar(kBarGate, kConsumers);
  if (warp != 0) return;
  GateRec mine = empty_rec();
  for (int bb = 0; bb < a.batch; ++bb) {
    const GateRec r = warp_merge(lane < kConsumerWarps ? gws[lane * a.batch + bb] : empty_rec());
    if (lane == bb) mine = r;
  }
  gate_publish(a, mine, lane);
}

// All consumer threads of a CTA that holds gate-problem units, after the CTA's outputs are
// written: the CTA's rows of that problem are one contiguous range [r0, r1) (still in L2).
// Every thread loads its strided share (up to kGateLoads values per batch row at once), takes
// the top-2 and S, T relative to its own max; warps merge (redux / shuffles), then warp 0
// merges the warps (one lane per warp) and publishes. gws: [kConsumerWarps][batch] in smem.
constexpr int kGateLoads = 8;
template <int MAXP>
__device__ __forceinline__ void gate_cta_reduce(const Args<MAXP>& a, const float* y, size_t ystride, int r0, int r1,
                                                GateRec* gws, int tid, int warp, int lane) {
  for (int bb = 0; bb < a.batch; ++bb) {
    const float* yr = y + (size_t)bb * ystride;
    GateRec r = empty_rec();
    for (int base = r0 + tid; base < r1; base += kGateLoads * kConsumers) {
      float v[kGateLoads];
#pragma unroll
      for (int j = 0; j < kGateLoads; ++j) {
        const int k = base + j * kConsumers;
        v[j] = (k < r1) ? __ldcg(yr + k) : -INFINITY;
      }
      GateRec q = empty_rec();
      float a1 = -INFINITY, a2 = -INFINITY;
      int j1 = 0x7fffffff, j2 = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < kGateLoads; ++j) {
        const int k = base + j * kConsumers;
        if (k < r1 && better(v[j], k, a2, j2)) {
          if (better(v[j], k, a1, j1)) {
            a2 = a1;
            j2 = j1;
            a1 = v[j];
            j1 = k;
          } else {
            a2 = v[j];
            j2 = k;
          }
        }
      }
      q.m = a1;
      q.i1 = j1;
      q.v2 = a2;
      q.i2 = j2;
      float S = 0.f, T = 0.f;
#pragma unroll
      for (int j = 0; j < kGateLoads; ++j) {
        if (base + j * kConsumers < r1) {
          const float d = v[j] - a1, e = __expf(d);
          S += e;
          T = fmaf(d, e, T);
        }
      }
      q.S = S;
      q.T = T;
      r = merge2(r, q);
    }
    r = warp_merge(r);
    if (lane == 0) gws[warp * a.batch + bb] = r;
  }
  gate_cta_finish(a, gws, warp, lane);
}

// Plane range [k0, k0 + np) read for block b, packed as k0 << 4 | np.
__device__ __forceinline__ int plane_range(int mode, const uint8_t* lv_from, const uint8_t* lv_to, int b) {
  const int lf = min((int)__ldg(lv_from + b), 4);
  if (mode == 0) return lf;
  const int lt = min((int)__ldg(lv_to + b), 4);
  return (lf << 4) | max(0, lt - lf);
}

// GATE: the logit gate is fused over problem a.gate_p's outputs (a separate instantiation,
// so the lane partials cost the plain kernel no registers).
template <int MAXP, int NT, bool GATE, bool LISTED>
__global__ void __launch_bounds__(kThreads, 1) plane_gemv_kernel(const __grid_constant__ Args<MAXP> a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t x_bar;  // staged activations have landed
  __shared__ Slot slots[kMaxSlots];
  __shared__ uint8_t lvc[kLevelCache];
  __shared__ int32_t bic[LISTED ? kListCache : 1];  // listed pass: block index of each unit
  __shared__ __align__(16) uint8_t zeros[160];
  __shared__ int s_ticket[kTeams];
  __shared__ int s_nslots;
  __shared__ int s_failed;  // a consumer warp gave up waiting for a stage

  pdl_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u_begin = a.cta_begin[blockIdx.x], u_end = a.cta_begin[blockIdx.x + 1];
  if (u_begin >= u_end) return;
  const int nunits = u_end - u_begin;
  // fused gate: this CTA holds gate-problem units; per consumer warp and batch row, its
  // partials (end of dynamic smem)
  const bool gate_cta = GATE && (int)blockIdx.x >= a.gate_cta0 && (int)blockIdx.x < a.gate_cta0 + a.gate_ncta;
  GateRec* const gws = reinterpret_cast<GateRec*>(smem + kSmemLimit - kConsumerWarps * a.batch * sizeof(GateRec));

  if (threadIdx.x < 40) reinterpret_cast<uint32_t*>(zeros)[threadIdx.x] = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kTeamWarps);
    }
    mbar_init(&x_bar, 1);
    fence_mbar_init();
    s_failed = 0;
  }
  if (warp == 0) {
    // Slot table: lane i fills slot i, the i-th (problem, slice) pair from the CTA's first one
    // (a multi-problem launch has one slice per problem); digit areas laid out back to back.
    const uint32_t base = smem_u32(smem + kStages * stage_bytes(NT));
    const int s0 = a.cta_slice[blockIdx.x] >> 7, nsl_cta = a.cta_slice[blockIdx.x] & 127;
    uint32_t carry = 0;
    int items = 0, n = 0;
    for (int i0 = 0; i0 < nsl_cta; i0 += 32) {
      const int i = i0 + lane;
      const bool live = i < nsl_cta;
      Slot sl;
      uint32_t bytes = 0;
      int nit = 0;
      if (live) {
        const int p = (a.nproblems == 1) ? 0 : s0 + i;
        const int j = (a.nproblems == 1) ? s0 + i : 0;
        const Problem& P = a.p[p];
        const int slice_start = P.unit_begin + j * P.nblocks;
        const int first = max(slice_start, u_begin);
        sl.p = p;
        sl.j = j;
        sl.u0 = first - u_begin;
        sl.u1 = min(u_end, slice_start + P.nblocks) - u_begin;
        sl.b0 = first - slice_start;
        sl.nblocks = P.nblocks;
        sl.ynb = P.ynb;
        sl.list = P.list;
        sl.G = P.G;
        sl.ngroups = slice_ng(P, j);
        sl.slices = P.slices;
        sl.gfirst = j * P.slice_groups;
        sl.stride = 128 * sl.ngroups + 16;
        sl.store = P.store;
        sl.lv_from = P.lv_from;
        sl.lv_to = P.lv_to;
        sl.x = P.x;
        sl.y = P.y;
        sl.partial = P.partial;
        sl.tickets = P.tickets;
        bytes = (uint32_t)(4 * a.batch * sl.stride + 8 * 4 * NT * sl.ngroups);
        nit = a.batch * sl.ngroups;
      }
      uint32_t incl = bytes;
      int iincl = nit;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        const int w = __shfl_up_sync(0xffffffffu, iincl, o);
        if (lane >= o) {
          incl += v;
          iincl += w;
        }
      }
      if (live) {
        sl.digits = base + carry + incl - bytes;
        sl.gconst = sl.digits + (uint32_t)(4 * a.batch * sl.stride);
        sl.it0 = items + iincl - nit;
        slots[i] = sl;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
      items += __shfl_sync(0xffffffffu, iincl, 31);
      n += __popc(__ballot_sync(0xffffffffu, live));
    }
    if (lane == 0) s_nslots = n;
  }
  __syncthreads();
  pdl_wait();  // everything above read only the parameters
  if (a.run_if != nullptr) {
    if (*reinterpret_cast<const volatile uint8_t*>(a.run_if) == 0) return;  // every thread reads the same byte
    if (blockIdx.x == 0 && threadIdx.x == 0 && a.runs != nullptr) atomicAdd(a.runs, 1u);
  }

  // Before any weight copy is in flight (they would queue ahead of these small reads): the
  // producer threads read the level bytes into the level cache while the consumer threads read
  // the activations. Producers then publish the cache with an arrive on kBarLevels and start
  // copying; consumers wait on it only once their digits are built.
  //
  // Team t (producer warp t and consumer warps 4t..4t+3) walks units t, t + kTeams, ... of the
  // range; both sides derive the same tile sequence from the slot table and the level cache,
  // so the only hand-offs are the full / empty barriers of the team's two stages.
  const int nsl = s_nslots;
  const int ditems = slots[nsl - 1].it0 + a.batch * slots[nsl - 1].ngroups;  // activation items
  const bool dmulti = ditems > 4 * kConsumerWarps;
  // staged: all activation rows fit the stage buffers, which stay idle until the digits are built
  const bool dstaged = dmulti && ditems * 256 <= kStages * stage_bytes(NT);
  if (warp >= kConsumerWarps) {
    // ---------------------------------------------------------------- producer warps
    {
      int si = 0;
      for (int k = threadIdx.x - kConsumers; k < nunits; k += 32 * kProducerWarps) {
        while (si + 1 < nsl && k >= slots[si].u1) ++si;
        const Slot& sl = slots[si];
        int b = sl.b0 + (k - sl.u0);
        if constexpr (LISTED) {
          b = sl.list[b];
          if (b < 0 || b >= sl.ynb) {  // the list lives on the device: checked here, skipped, reported
            atomicExch(&g_error, 5);
            b = -1;
          }
          bic[k] = b;
        }
        lvc[k] = b < 0 ? (uint8_t)kSkipUnit : (uint8_t)plane_range(a.mode, sl.lv_from, sl.lv_to, b);
      }
    }
    named_bar(kBarProducers, 32 * kProducerWarps);
    bar_arrive(kBarLevels, kThreads);
    if (dmulti) {
      named_bar(kBarX, kThreads);
      // the staged activations never arrived: issue nothing into stages they may still reach
      if (s_failed) return;
    }
    if (lane != 0) return;
    const int team = warp - kConsumerWarps;
    int issued = 0, si = 0;
    for (int k = team; k < nunits; k += kTeams) {
      while (si + 1 < nsl && k >= slots[si].u1) ++si;
      const Slot& sl = slots[si];
      const int b = LISTED ? bic[k] : sl.b0 + (k - sl.u0);
      const int pr = (int)lvc[k];
      const int k0 = pr >> 4, np = pr & 15;
      if (np == 0 || (LISTED && pr == kSkipUnit)) continue;
      const int tgm = tile_groups(np, NT);
      const int ngs = sl.ngroups;
      const int G = sl.G;
      const uint8_t* blk = sl.store + (size_t)b * 8448u * G;
      for (int g0 = 0; g0 < ngs; g0 += tgm) {
        const int tg = min(tgm, ngs - g0);
        const int s = kTeamStages * team + (issued % kTeamStages);
        if (issued >= kTeamStages &&
            !mbar_wait(&empty_bar[s], (uint32_t)((issued / kTeamStages - 1) & 1))) {
          atomicExch(&g_error, 1);
          return;
        }
        uint8_t* st = smem + s * stage_bytes(NT);
        const int gg = sl.gfirst + g0;
        const uint32_t bytes = 256u * tg + 2048u * tg * np;
        mbar_expect_tx(&full_bar[s], bytes);
        if (tg == G && k0 == 0) {
          bulk_g2s(st, blk, bytes, &full_bar[s]);  // the whole depth-d prefix of the block
        } else {
          bulk_g2s(st, blk + 256u * gg, 256u * tg, &full_bar[s]);
          for (int kk = 0; kk < np; ++kk)
            bulk_g2s(st + 256 * tg + 2048 * tg * kk, blk + 256u * G + 2048u * ((size_t)G * (k0 + kk) + gg),
                     2048u * tg, &full_bar[s]);
        }
        ++issued;
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumer warps
  // 1. activation digits of every (problem, slice) the range touches
  if (dstaged) {
    if (threadIdx.x == 0) stage_x(slots, nsl, a.batch, smem, &x_bar, ditems);
    // warp-uniform outcome: a warp whose wait ran out converts nothing and flags the CTA
    // before its arrive, so the producers (after kBarX) and every consumer (after kBarLevels)
    // see the flag and the CTA skips its tiles
    if (__all_sync(0xffffffffu, mbar_wait(&x_bar, 0u))) {
      convert_staged(slots, nsl, a.batch, 4 * NT, smem, threadIdx.x, kConsumers, ditems);
    } else if (lane == 0) {
      atomicExch(&g_error, 3);
      s_failed = 1;
    }
    bar_arrive(kBarX, kThreads);  // the stage buffers are free for the weight stream
  } else {
    build_digits(slots, nsl, a.batch, 4 * NT, threadIdx.x, kConsumers, ditems, dmulti);
  }
  named_bar(kBarLevels, kThreads);  // every consumer's digits, and the producers' level cache

  // 2. team loop
  const int team = warp / kTeamWarps, mt = warp % kTeamWarps;
  const int tt = threadIdx.x % kTeamThreads;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * mt + g;
  const uint32_t smem_base = smem_u32(smem);
  uint32_t dlane[NT], dstep[NT], gc_lane = 0;
  int cur_slot = -1, si = 0, used = 0;
  // failed: a wait of this warp ran out (or the staged activations never arrived, CTA-uniform
  // here). From then on the warp skips its waits and its math but still takes every team
  // barrier below, so no named barrier is left short of a participant; the outputs are not
  // valid and the error word says so.
  bool failed = s_failed != 0;
  for (int k = team; k < nunits; k += kTeams) {
    while (si + 1 < nsl && k >= slots[si].u1) ++si;
    const Slot& sl = slots[si];
    const int b = LISTED ? bic[k] : sl.b0 + (k - sl.u0);
    const int pr = (int)lvc[k];
    if (LISTED && pr == kSkipUnit) continue;
    const int k0 = pr >> 4, np = pr & 15;
    const size_t ystride = (size_t)64 * (LISTED ? sl.ynb : sl.nblocks);
    const int row_base = 64 * b + 16 * mt;
    float* const y = sl.y;
    if (np == 0) {  // ZERO block (depth mode): its rows are 0; a residual adds nothing
      if (a.mode == 0 && sl.j == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int bb = 4 * nt + t;
          if (bb < a.batch) {
            y[(size_t)bb * ystride + row_base + g] = 0.f;
            y[(size_t)bb * ystride + row_base + g + 8] = 0.f;
          }
        }
      }
      continue;
    }
    if (si != cur_slot) {
      cur_slot = si;
      gc_lane = sl.gconst + 8u * (uint32_t)(t * sl.ngroups);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int row = 8 * nt + g;
        const bool liveb = row < 4 * a.batch;
        dlane[nt] = liveb ? sl.digits + (uint32_t)(row * sl.stride + 32 * t) : smem_u32(zeros + 32 * t);
        dstep[nt] = liveb ? 128u : 0u;
      }
    }
    const int gstride = sl.ngroups;
    const float cfac = cfac_of(k0, np);
    float acc[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
    const int tgm = tile_groups(np, NT);
    for (int g0 = 0; g0 < sl.ngroups; g0 += tgm) {
      const int tg = min(tgm, sl.ngroups - g0);
      const int s = kTeamStages * team + (used % kTeamStages);
      ++used;
      if (failed) continue;
      if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[s], (uint32_t)(((used - 1) / kTeamStages) & 1)))) {
        if (lane == 0) {
          atomicExch(&g_error, 2);
          s_failed = 1;
        }
        failed = true;
        continue;
      }
      dispatch_tile<NT>(k0, np, smem_base + s * stage_bytes(NT), tg, dlane, dstep, gc_lane, gstride, g0, cfac, r0, t,
                        acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }

    // ---- unit done: this warp's 16 rows are final (or a slice partial). Lane t holds digit
    // pair t & 1 of batch row 2 nt + t / 2; the pairs' sums meet in one shuffle and the even
    // lane writes.
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      acc[nt][0] += __shfl_xor_sync(0xffffffffu, acc[nt][0], 1);
      acc[nt][1] += __shfl_xor_sync(0xffffffffu, acc[nt][1], 1);
    }
    if (sl.slices == 1) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int bb = 2 * nt + (t >> 1);
        if ((t & 1) == 0 && bb < a.batch) {
          float* y0 = y + (size_t)bb * ystride + row_base + g;
          if (a.mode == 1) {
            // the residual adds to y where y lives (a reduction in L2, no load on the team's
            // path); each output is added to once per pass
            red_add_f32(y0, acc[nt][0]);
            red_add_f32(y0 + 8, acc[nt][1]);
          } else {
            y0[0] = acc[nt][0];
            y0[8] = acc[nt][1];
          }
        }
      }
    } else {
      // partial for this slice; the last team to finish the block adds the slices in order
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int bb = 2 * nt + (t >> 1);
        if ((t & 1) == 0 && bb < a.batch) {
          float* pp = sl.partial + (((size_t)sl.j * sl.nblocks + b) * a.batch + bb) * 64 + 16 * mt + g;
          pp[0] = acc[nt][0];
          pp[8] = acc[nt][1];
        }
      }
      // The barrier orders the team's partial stores before thread 0's acquire-release ticket
      // (release is cumulative); the last team's reads follow the ticket's acquire.
      named_bar(kBarTeam0 + team, kTeamThreads);
      if (tt == 0) s_ticket[team] = (int)atom_add_acq_rel(&sl.tickets[b], 1u);
      named_bar(kBarTeam0 + team, kTeamThreads);
      if (s_ticket[team] == sl.slices - 1) {
        if (a.batch * 64 <= kTeamThreads) {  // one output per thread at most
          const int e = tt;
          if (e < a.batch * 64) {
            float sum = 0.f;
#pragma unroll 4
            for (int jj = 0; jj < sl.slices; ++jj)
              sum += __ldcg(sl.partial + (((size_t)jj * sl.nblocks + b) * a.batch + e / 64) * 64 + e % 64);
            float* yy = y + (size_t)(e / 64) * ystride + 64 * b + e % 64;
            if (a.mode == 0)
              *yy = sum;
            else
              red_add_f32(yy, sum);
          }
        } else
        // each thread's outputs (up to kRed) and slices: every load is issued before the sums
        for (int e0 = tt; e0 < a.batch * 64; e0 += kRed * kTeamThreads) {
          float sum[kRed];
#pragma unroll
          for (int q = 0; q < kRed; ++q) sum[q] = 0.f;
          for (int jj = 0; jj < sl.slices; ++jj) {
            float v[kRed];
#pragma unroll
            for (int q = 0; q < kRed; ++q) {
              const int e = e0 + q * kTeamThreads;
              v[q] = (e < a.batch * 64)
                         ? __ldcg(sl.partial + (((size_t)jj * sl.nblocks + b) * a.batch + e / 64) * 64 + e % 64)
                         : 0.f;
            }
#pragma unroll
            for (int q = 0; q < kRed; ++q) sum[q] += v[q];
          }
#pragma unroll
          for (int q = 0; q < kRed; ++q) {
            const int e = e0 + q * kTeamThreads;
            if (e < a.batch * 64) {
              float* yy = y + (size_t)(e / 64) * ystride + 64 * b + e % 64;
              if (a.mode == 0)
                *yy = sum[q];
              else
                red_add_f32(yy, sum[q]);
            }
          }
        }
        if (tt == 0) sl.tickets[b] = 0u;
      }
      named_bar(kBarTeam0 + team, kTeamThreads);
    }
  }
  if constexpr (GATE) {
    if (gate_cta) {
      // every consumer warp has written its outputs (this barrier also orders them)
      named_bar(kBarGate, kConsumers);
      if (s_failed) return;
      const Problem& P = a.p[a.gate_p];
      const int b0 = max(u_begin, P.unit_begin) - P.unit_begin;
      const int b1 = min(u_end, P.unit_begin + P.nblocks) - P.unit_begin;
      gate_cta_reduce(a, P.y, (size_t)64 * P.nblocks, 64 * b0, 64 * b1, gws, threadIdx.x, warp, lane);
    }
  }
}

// ---------------------------------------------------------------- host side

struct Plan {
  int slices, slice_groups;
};

// N-tiles of the products: two digit pairs per batch row, four pairs per 8-column N-tile.
__host__ __device__ constexpr int ntiles(int batch) { return (batch + 1) / 2; }

static size_t slot_bytes(int batch, int ngroups) {
  const int nt = ntiles(batch);
  return (size_t)4 * batch * (128 * ngroups + 16) + (size_t)8 * 4 * nt * ngroups;
}

// Widest column slice (in 128-column groups) whose digits fit in one slot.
static int max_groups_fit(int batch, long budget) {
  const int nt = ntiles(batch);
  const long avail = budget - 64L * batch;
  return (int)std::max(1L, avail / (512L * batch + 32L * nt));
}

// Column split for a single layer: enough units to fill the GPU, slices of whole
// groups, and a slice narrow enough for the activation digits to fit in smem.
static Plan plan_single(int nblocks, int G, int batch, int nsm) {
  Plan pl;
  const int max_sg = max_groups_fit(batch, digit_budget(ntiles(batch)));
  const int s_mem = (G + max_sg - 1) / max_sg;
  const int s_fill = (2 * nsm + nblocks - 1) / nblocks;
  int s = std::max(s_mem, std::min(s_fill, std::max(1, G / 4)));
  s = std::min(s, G);
  pl.slice_groups = (G + s - 1) / s;
  pl.slices = (G + pl.slice_groups - 1) / pl.slice_groups;
  return pl;
}

static size_t workspace_for(const Plan& pl, int nblocks, int batch) {
  if (pl.slices <= 1) return 0;
  const size_t tickets = ((size_t)nblocks * 4 + 255) / 256 * 256;
  return tickets + (size_t)pl.slices * nblocks * batch * 64 * 4;
}

// Contiguous cost-balanced unit ranges, one per CTA (cost ~ columns read). A range is also
// closed early when the digits of its distinct (problem, slice) pairs would overflow shared
// memory, at kMaxSlots pairs, or at the level-cache size; after every cut the cost still to
// place is spread evenly over the ranges still to make, so an early cut does not leave a later
// range oversized. Cuts can still make more ranges than SMs (a second, partial wave) when
// memory forces more than that. The fused gate's epilogue (a reduction of the CTA's logits and
// a publish, a few us) is charged to the gate problem's units, so the CTAs holding them get
// fewer weight bytes. The weight is measured: on the 197-layer decode pass at batch 1 the fused
// launch takes 58.5 us at 1.08, 56.1 us at 1.25 and 57.3 / 58.5 us at 1.35 / 1.5 (the pass
// without the gate: 54.0 us).
constexpr double kGateUnitWeight = 1.25;
// A (problem, slice) pair's activation digits cost a CTA's prologue about as much as 7 groups.
constexpr double kSlotCost = 7.0;

template <int MAXP>
static double unit_weight(const Args<MAXP>& a, int i) {
  return i == a.gate_p ? kGateUnitWeight : 1.0;
}

template <int MAXP>
static bool partition(Args<MAXP>& a, int nsm, size_t budget) {
  double total = 0;
  int pairs = 0;
  for (int i = 0; i < a.nproblems; ++i) {
    total += (double)a.p[i].nblocks * a.p[i].G * unit_weight(a, i);
    pairs += a.p[i].slices;
  }
  const Problem& L = a.p[a.nproblems - 1];
  const int units = L.unit_begin + L.nblocks * L.slices;
  const int target = std::max(1, std::min(nsm, units));
  total += kSlotCost * (pairs + target - 1);  // about one slot per pair plus one per cut
  double per_cta = total / target;
  double start = 0;  // cumulative cost where the current range began
  int n = 0;
  a.cta_begin[0] = 0;
  a.cta_slice[0] = 0;
  double acc = 0;      // cumulative cost from the first unit
  size_t dig = 0;      // digit bytes of the current range
  int nslots = 0, count = 0;
  for (int i = 0; i < a.nproblems; ++i) {
    const Problem& P = a.p[i];
    for (int j = 0; j < P.slices; ++j) {
      const int ng = std::min(P.slice_groups, P.G - j * P.slice_groups);
      const size_t sb = slot_bytes(a.batch, ng);
      const double cost = (double)ng * unit_weight(a, i);
      for (int b = 0; b < P.nblocks; ++b) {
        const int u = P.unit_begin + j * P.nblocks + b;
        bool cut = false;
        if (count > 0) {
          if (n + 1 < target && acc + 0.5 * cost - start > per_cta) cut = true;
          if (b == 0 && (dig + sb > budget || nslots == kMaxSlots)) cut = true;
          if (count == (a.listed ? kListCache : kLevelCache)) cut = true;
        }
        if (cut) {
          if (n + 1 >= kMaxCtas) return false;
          a.cta_slice[n] |= nslots;
          a.cta_begin[++n] = u;
          a.cta_slice[n] = ((a.nproblems == 1) ? j : i) << 7;
          dig = 0;
          nslots = 0;
          count = 0;
          start = acc;
          per_cta = (total - acc) / std::max(1, target - n);
        }
        if (b == 0 || count == 0) {
          dig += sb;
          ++nslots;
          acc += kSlotCost;
        }
        acc += cost;
        ++count;
      }
    }
  }
  a.cta_slice[n] |= nslots;
  a.cta_begin[++n] = units;
  a.ncta = n;
  return true;
}

template <int MAXP, int NT, bool GATE, bool LISTED = false>
static fl_status launch(const Args<MAXP>& a, cudaStream_t st) {
  const size_t smem = (size_t)kSmemLimit;
  auto kern = plane_gemv_kernel<MAXP, NT, GATE, LISTED>;
  FL_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                "cudaFuncSetAttribute(plane_gemv)");
  FL_CHECK_CUDA(launch_pdl(kern, dim3(a.ncta), dim3(kThreads), smem, st, 1, a), "launch plane_gemv");
  return FL_OK;
}

template <int MAXP, bool GATE, bool LISTED>
static fl_status launch_by_batch(const Args<MAXP>& a, cudaStream_t st) {
  switch (ntiles(a.batch)) {
    case 1: return launch<MAXP, 1, GATE, LISTED>(a, st);
    case 2: return launch<MAXP, 2, GATE, LISTED>(a, st);
    case 3: return launch<MAXP, 3, GATE, LISTED>(a, st);
    case 4: return launch<MAXP, 4, GATE, LISTED>(a, st);
    case 5: return launch<MAXP, 5, GATE, LISTED>(a, st);
    case 6: return launch<MAXP, 6, GATE, LISTED>(a, st);
    case 7: return launch<MAXP, 7, GATE, LISTED>(a, st);
    default: return launch<MAXP, 8, GATE, LISTED>(a, st);
  }
}

static fl_status launch_nt_gate(const Args<FL_MAX_PROBLEMS>& a, cudaStream_t st) {
  return launch_by_batch<FL_MAX_PROBLEMS, true, false>(a, st);
}

template <int MAXP>
static fl_status launch_nt(const Args<MAXP>& a, cudaStream_t st) {
  if constexpr (MAXP > 1) {
    if (a.listed) return launch_by_batch<MAXP, false, true>(a, st);
  }
  return launch_by_batch<MAXP, false, false>(a, st);
}

static fl_status check_weight(const fl_plane_weight* w, const char* what) {
  if (!w) return fail(FL_ERR_ARG, "%s: weight descriptor is NULL", what);
  if (!w->store) return fail(FL_ERR_ARG, "%s: plane store pointer is NULL", what);
  if (w->out <= 0 || w->in <= 0 || w->out % 64 || w->in % 128)
    return fail(FL_ERR_SHAPE, "%s: out=%d in=%d (need out %% 64 == 0, in %% 128 == 0)", what, w->out, w->in);
  if (!aligned16(w->store)) return fail(FL_ERR_ALIGN, "%s: plane store not 16-byte aligned", what);
  return FL_OK;
}

// Every host-side check of a single-layer call, then its launch parameters in `a`; nothing is
// enqueued.
static fl_status prepare_single(Args<1>& a, const fl_plane_weight* w, const uint8_t* lv_from, const uint8_t* lv_to,
                                const uint16_t* x, int batch, float* y, void* ws, size_t ws_bytes, int mode,
                                const char* what) {
  fl_status st = check_weight(w, what);
  if (st != FL_OK) return st;
  if (!lv_from || !x || !y || (mode == 1 && !lv_to)) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
  if (reinterpret_cast<uintptr_t>(y) & 3u) return fail(FL_ERR_ALIGN, "%s: y not 4-byte aligned", what);
  if (batch < 1 || batch > FL_MAX_GEMV_BATCH)
    return fail(FL_ERR_SHAPE, "%s: batch=%d (1..%d)", what, batch, FL_MAX_GEMV_BATCH);
  if (batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..%d on this path)", what, batch, FL_MAX_BATCH);
  if (!aligned16(x)) return fail(FL_ERR_ALIGN, "%s: x not 16-byte aligned", what);
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  const int nblocks = w->out / 64, G = w->in / 128;
  Plan pl = plan_single(nblocks, G, batch, nsm);
  const size_t need = workspace_for(pl, nblocks, batch);
  if (need > 0 && (!ws || ws_bytes < need))
    return fail(FL_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", what, ws ? ws_bytes : (size_t)0, need);
  if (need > 0 && !aligned16(ws)) return fail(FL_ERR_ALIGN, "%s: workspace not 16-byte aligned", what);
  a.nproblems = 1;
  a.batch = batch;
  a.mode = mode;
  a.gate_p = -1;
  a.run_if = nullptr;
  a.runs = nullptr;
  a.gate_partial = nullptr;
  a.gate_index_base = 0;
  a.listed = 0;
  Problem& P = a.p[0];
  P.store = w->store;
  P.lv_from = lv_from;
  P.lv_to = lv_to;
  P.x = x;
  P.y = y;
  P.nblocks = nblocks;
  P.ynb = nblocks;
  P.list = nullptr;
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
  if (!partition(a, nsm, (size_t)digit_budget(ntiles(batch))))
    return fail(FL_ERR_SHAPE, "%s: layer too large for one launch", what);
  return FL_OK;
}

static fl_status single(const fl_plane_weight* w, const uint8_t* lv_from, const uint8_t* lv_to, const uint16_t* x,
                        int batch, float* y, void* ws, size_t ws_bytes, void* stream, int mode,
                        const char* what) {
  if (batch >= 1 && batch <= FL_MAX_GEMV_BATCH && tc_takes(batch)) {
    fl_status st = check_weight(w, what);
    if (st != FL_OK) return st;
    if (!lv_from || !x || !y || (mode == 1 && !lv_to)) return fail(FL_ERR_ARG, "%s: NULL pointer argument", what);
    if (reinterpret_cast<uintptr_t>(y) & 3u) return fail(FL_ERR_ALIGN, "%s: y not 4-byte aligned", what);
    if (!aligned16(x)) return fail(FL_ERR_ALIGN, "%s: x not 16-byte aligned", what);
    return tc_single(w, lv_from, lv_to, x, batch, y, ws, ws_bytes, stream, mode, what);
  }
  static thread_local Args<1> a;
  const fl_status st = prepare_single(a, w, lv_from, lv_to, x, batch, y, ws, ws_bytes, mode, what);
  if (st != FL_OK) return st;
  return launch_nt(a, static_cast<cudaStream_t>(stream));
}

}  // namespace gemv
}  // namespace fl

using namespace fl;

extern "C" size_t fl_gemv_workspace_bytes(int out, int in, int batch) {
  if (out <= 0 || in <= 0 || out % 64 || in % 128 || batch < 1 || batch > FL_MAX_GEMV_BATCH) return 0;
  if (tc_takes(batch)) return tc_workspace_bytes(out, in, batch);
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

namespace fl {
namespace gemv {

constexpr size_t kGateTicketBytes = 256;
constexpr size_t kGateWorkspaceBytes = kGateTicketBytes + (size_t)kMaxCtas * FL_MAX_BATCH * sizeof(GateRec);

static fl_status batched(const fl_gemv_problem* problems, int n, int batch, int mode, const fl_gate_spec* gate,
                         const uint8_t* run_if, uint32_t* runs, void* stream, const char* what,
                         const int32_t* const* lists = nullptr, const int* counts = nullptr,
                         fl_gate_partial* partial = nullptr, int index_base = 0) {
  if (!problems) return fail(FL_ERR_ARG, "%s: problems is NULL", what);
  if (n < 1 || n > FL_MAX_PROBLEMS) return fail(FL_ERR_ARG, "%s: n=%d (1..%d)", what, n, FL_MAX_PROBLEMS);
  if (mode != 0 && mode != 1) return fail(FL_ERR_ARG, "%s: mode=%d (0 depth, 1 residual)", what, mode);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  static thread_local Args<FL_MAX_PROBLEMS> a;
  a.nproblems = n;
  a.batch = batch;
  a.mode = mode;
  a.gate_p = -1;
  a.run_if = run_if;
  a.runs = runs;
  a.gate_partial = reinterpret_cast<GateRec*>(partial);
  a.gate_index_base = index_base;
  a.listed = lists != nullptr ? 1 : 0;
  if (reinterpret_cast<uintptr_t>(runs) & 3u) return fail(FL_ERR_ALIGN, "%s: runs not 4-byte aligned", what);
  if (lists != nullptr && (counts == nullptr || gate != nullptr))
    return fail(FL_ERR_ARG, "%s: a listed pass needs counts and has no gate", what);
  size_t budget = (size_t)digit_budget(ntiles(batch));
  if (gate) {
    if (gate->problem < 0 || gate->problem >= n)
      return fail(FL_ERR_ARG, "%s: gate problem %d not in 0..%d", what, gate->problem, n - 1);
    if ((!partial && (!gate->entropy || !gate->margin || !gate->top2 || !gate->escalate)) || !gate->workspace)
      return fail(FL_ERR_ARG, "%s: gate output or workspace pointer is NULL", what);
    if (partial && (!aligned16(partial) || index_base < 0 ||
                    (long long)index_base + problems[gate->problem].w.out > (1LL << 24)))
      return fail(FL_ERR_ARG, "%s: partial must be 16-byte aligned, index_base + out below 2^24", what);
    if (gate->workspace_bytes < kGateWorkspaceBytes)
      return fail(FL_ERR_WORKSPACE, "%s: gate workspace %zu bytes, need %zu", what, gate->workspace_bytes,
                  kGateWorkspaceBytes);
    if (!aligned16(gate->workspace)) return fail(FL_ERR_ALIGN, "%s: gate workspace not 16-byte aligned", what);
    if (!partial && ((reinterpret_cast<uintptr_t>(gate->entropy) | reinterpret_cast<uintptr_t>(gate->margin) |
                      reinterpret_cast<uintptr_t>(gate->top2)) & 3u))
      return fail(FL_ERR_ALIGN, "%s: gate entropy, margin and top2 must be 4-byte aligned", what);
    a.gate_p = gate->problem;
    a.tau_h = gate->tau_h;
    a.tau_m = gate->tau_m;
    a.entropy = gate->entropy;
    a.margin = gate->margin;
    a.top2 = gate->top2;
    a.escalate = gate->escalate;
    a.gate_ticket = static_cast<uint32_t*>(gate->workspace);
    a.gate_part = reinterpret_cast<GateRec*>(static_cast<uint8_t*>(gate->workspace) + kGateTicketBytes);
    budget -= (size_t)kConsumerWarps * batch * sizeof(GateRec);
  }
  int unit = 0, np = 0;  // np: problems launched (a listed pass drops those with no listed block)
  for (int i = 0; i < n; ++i) {
    const fl_gemv_problem& q = problems[i];
    fl_status st = check_weight(&q.w, what);
    if (st != FL_OK) return st;
    if (!q.levels || !q.x || !q.y || (mode == 1 && !q.to_levels))
      return fail(FL_ERR_ARG, "%s: problem %d has a NULL pointer", what, i);
    if (reinterpret_cast<uintptr_t>(q.y) & 3u) return fail(FL_ERR_ALIGN, "%s: problem %d y not 4-byte aligned", what, i);
    if (!aligned16(q.x)) return fail(FL_ERR_ALIGN, "%s: problem %d x not 16-byte aligned", what, i);
    const int G = q.w.in / 128;
    if (G > max_groups_fit(batch, (long)budget))
      return fail(FL_ERR_SHAPE, "%s: problem %d in=%d too wide for batch %d in one launch (in <= %d)", what, i,
                  q.w.in, batch, 128 * max_groups_fit(batch, (long)budget));
    int units = q.w.out / 64;
    if (lists != nullptr) {
      if (counts[i] < 0 || counts[i] > q.w.out / 64)
        return fail(FL_ERR_ARG, "%s: problem %d lists %d blocks (0..%d)", what, i, counts[i], q.w.out / 64);
      if (counts[i] > 0 && lists[i] == nullptr) return fail(FL_ERR_ARG, "%s: problem %d list is NULL", what, i);
      if (reinterpret_cast<uintptr_t>(lists[i]) & 3u)
        return fail(FL_ERR_ALIGN, "%s: problem %d list not 4-byte aligned", what, i);
      units = counts[i];
      if (units == 0) continue;
    }
    Problem& P = a.p[np++];
    P.store = q.w.store;
    P.lv_from = q.levels;
    P.lv_to = q.to_levels;
    P.x = q.x;
    P.y = q.y;
    P.partial = nullptr;
    P.tickets = nullptr;
    P.nblocks = units;
    P.ynb = q.w.out / 64;
    P.list = lists != nullptr ? lists[i] : nullptr;
    P.G = G;
    P.slices = 1;
    P.slice_groups = G;
    P.unit_begin = unit;
    unit += P.nblocks;
  }
  if (np == 0) return FL_OK;  // a listed pass with nothing listed: no launch
  a.nproblems = np;
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  if (!partition(a, nsm, budget)) return fail(FL_ERR_SHAPE, "%s: problems too large for one launch", what);
  if (gate) {
    const int ub = a.p[a.gate_p].unit_begin, ue = ub + a.p[a.gate_p].nblocks;
    a.gate_cta0 = -1;
    a.gate_ncta = 0;
    for (int c = 0; c < a.ncta; ++c)
      if (a.cta_begin[c] < ue && a.cta_begin[c + 1] > ub) {
        if (a.gate_cta0 < 0) a.gate_cta0 = c;
        ++a.gate_ncta;
      }
    return launch_nt_gate(a, static_cast<cudaStream_t>(stream));
  }
  return launch_nt(a, static_cast<cudaStream_t>(stream));
}

}  // namespace gemv
}  // namespace fl

extern "C" fl_status fl_gemv_batched(const fl_gemv_problem* problems, int n, int batch, int mode, void* stream) {
  return gemv::batched(problems, n, batch, mode, nullptr, nullptr, nullptr, stream, "fl_gemv_batched");
}

extern "C" fl_status fl_gemv_batched_listed(const fl_gemv_problem* problems, const int32_t* const* lists,
                                            const int* counts, int n, int batch, int mode, void* stream) {
  if (!lists || !counts) return fail(FL_ERR_ARG, "fl_gemv_batched_listed: lists or counts is NULL");
  return gemv::batched(problems, n, batch, mode, nullptr, nullptr, nullptr, stream, "fl_gemv_batched_listed", lists,
                       counts);
}

extern "C" size_t fl_gemv_gate_workspace_bytes(int batch) {
  if (batch < 1 || batch > FL_MAX_BATCH) return 0;
  return gemv::kGateWorkspaceBytes;
}

extern "C" fl_status fl_gemv_batched_gate(const fl_gemv_problem* problems, int n, int batch, int mode,
                                          const fl_gate_spec* gate, void* stream) {
  if (!gate) return fail(FL_ERR_ARG, "fl_gemv_batched_gate: gate spec is NULL");
  return gemv::batched(problems, n, batch, mode, gate, nullptr, nullptr, stream, "fl_gemv_batched_gate");
}

extern "C" fl_status fl_gemv_batched_gate_if(const fl_gemv_problem* problems, int n, int batch, int mode,
                                             const fl_gate_spec* gate, const uint8_t* run_if, uint32_t* runs,
                                             void* stream) {
  const char* what = "fl_gemv_batched_gate_if";
  if (!gate) return fail(FL_ERR_ARG, "%s: gate spec is NULL", what);
  if (!run_if) return fail(FL_ERR_ARG, "%s: run_if is NULL", what);
  return gemv::batched(problems, n, batch, mode, gate, run_if, runs, stream, what);
}

extern "C" fl_status fl_gemv_batched_gate_partial(const fl_gemv_problem* problems, int n, int batch, int mode,
                                                  const fl_gate_spec* gate, const uint8_t* run_if, uint32_t* runs,
                                                  int index_base, fl_gate_partial* partial, void* stream) {
  const char* what = "fl_gemv_batched_gate_partial";
  if (!gate) return fail(FL_ERR_ARG, "%s: gate spec is NULL", what);
  if (!partial) return fail(FL_ERR_ARG, "%s: partial is NULL", what);
  if (gate->problem < 0 || gate->problem >= n || !problems)
    return fail(FL_ERR_ARG, "%s: gate problem %d not in 0..%d", what, gate->problem, n - 1);
  return gemv::batched(problems, n, batch, mode, gate, run_if, runs, stream, what, nullptr, nullptr, partial,
                       index_base);
}

// ---------------------------------------------------------------- failure detection
namespace fl {
namespace gemv {

// Reads and clears the error word (-1 if that fails).
int take_device_error() {
  int v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_error, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0 && cudaMemcpyToSymbol(g_error, &z, sizeof(int)) != cudaSuccess) return -1;
  return v;
}

// One thread waits on a barrier that expects an arrival nobody makes, with the given deadline
// (the same bounded wait as the kernels' stage barriers, shorter).
__global__ void selftest_timeout_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait(&bar, 0u, limit_ns)) atomicExch(&g_error, 4);
}

}  // namespace gemv
}  // namespace fl

extern "C" fl_status fl_selftest_wait_timeout(void* stream) {
  FL_CHECK_CUDA(launch_pdl(gemv::selftest_timeout_kernel, dim3(1), dim3(1), 0, static_cast<cudaStream_t>(stream), 1,
                           (uint64_t)1000000u),
                "launch selftest_timeout");
  return FL_OK;
}

// ---------------------------------------------------------------- allocation-free variant
// The column-split scratch of fl_gemv_depth_static: one fixed array in the device image
// (tickets first, then the slice partials, as in a caller workspace). Its device address is
// looked up once per device, with that device current, on the first call there.
namespace fl {
namespace gemv {

static __device__ __align__(256) uint8_t g_static_scratch[FL_GEMV_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
static std::mutex g_static_mu;
static void* g_static_ptr[kMaxDevices];

static fl_status static_scratch(void** ptr, const char* what) {
  int dev = -1;
  FL_CHECK_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FL_ERR_CUDA, "%s: device %d out of range", what, dev);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_static_ptr[dev] = p;
  }
  *ptr = g_static_ptr[dev];
  return FL_OK;
}

}  // namespace gemv
}  // namespace fl

extern "C" fl_status fl_gemv_depth_static(const fl_plane_weight* w, const uint8_t* levels, const uint16_t* x,
                                          int batch, float* y, void* stream) {
  const char* what = "fl_gemv_depth_static";
  fl_status st = gemv::check_weight(w, what);
  if (st != FL_OK) return st;
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  const int nblocks = w->out / 64;
  const gemv::Plan pl = gemv::plan_single(nblocks, w->in / 128, batch, nsm);
  const size_t need = gemv::workspace_for(pl, nblocks, batch);
  if (need > (size_t)FL_GEMV_STATIC_SCRATCH_BYTES)
    return fail(FL_ERR_WORKSPACE,
                "%s: out=%d in=%d batch=%d needs %zu bytes of scratch, the built-in array holds %zu "
                "(use fl_gemv_depth with a caller workspace)",
                what, w->out, w->in, batch, need, (size_t)FL_GEMV_STATIC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (need > 0) {
    st = gemv::static_scratch(&scratch, what);
    if (st != FL_OK) return st;
  }
  static thread_local gemv::Args<1> a;
  st = gemv::prepare_single(a, w, levels, nullptr, x, batch, y, scratch,
                            need > 0 ? (size_t)FL_GEMV_STATIC_SCRATCH_BYTES : 0, 0, what);
  if (st != FL_OK) return st;  // rejected before anything is enqueued: the shared array is untouched
  if (need > 0) {
    // the split's tickets start at zero; the partials are written before they are read
    const size_t tickets = ((size_t)nblocks * 4 + 255) / 256 * 256;
    FL_CHECK_CUDA(cudaMemsetAsync(scratch, 0, tickets, static_cast<cudaStream_t>(stream)),
                  "cudaMemsetAsync(static scratch tickets)");
  }
  return gemv::launch_nt(a, static_cast<cudaStream_t>(stream));
}
