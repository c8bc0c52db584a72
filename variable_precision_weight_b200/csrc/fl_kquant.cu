// K-quant fused dequant GEMV ("v0.3, quantized on disk, quantized in memory":
// native Q4_K and Q6_K kernels that keep the weights compressed and
// dequantize only at block granularity inside the product; per-tensor
// dispatch, unsupported types fail).
//
//   Q4_K:  y[t][r] = sum_sb sum_j ( d sc_j sum_{c in j} q_c x_c  -  dmin mn_j sum_{c in j} x_c )
//   Q6_K:  y[t][r] = sum_sb sum_j   d sc_j sum_{c in j} (q_c - 32) x_c
//
// Same B200 structure as the plane-store GEMV: one persistent CTA per SM, a
// producer warp whose 32 lanes issue per-row 1-D bulk copies of a tile (64
// rows x a few super-blocks) into a 4-stage shared-memory ring, and eight
// consumer warps (4 m-tiles x 2 super-block parities). Codes become u8
// tensor-core operands with one or two mask/shift operations per four
// weights (the record layouts are built for it); each sub-block is one
// mma.sync (m16n8k32 for Q4_K's 32-weight sub-blocks, m16n8k16 for Q6_K's
// 16-weight ones) against the activations' int8 digits; the sub-block scale
// is applied to the int32 result with an integer multiply-add, and each
// 128-column half of a super-block is converted to fp32 once.
#include <algorithm>

#include "fl_common.cuh"

namespace fl {
namespace kq {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kConsumers + 32;
constexpr int kStages = 4;
constexpr int kStageBytes = 37888;
constexpr int kMaxCtas = 512;
constexpr int kSmemLimit = 232448 - 6144;  // opt-in shared memory per block on B200, less static use
constexpr int kQ4Tsb = 4;          // super-blocks per Q4_K tile
constexpr int kQ4Slot = 592;       // bytes per row in a Q4_K tile (4 records + 16 B pad against bank conflicts)
constexpr int kQ6Tsb = 2;          // super-blocks per Q6_K tile
constexpr int kQ6Slot = 432;       // bytes per row in a Q6_K tile (2 records, 16-byte rounded copy)

struct Problem {
  const uint8_t* blocks;
  const uint16_t* x;
  float* y;
  float* partial;
  uint32_t* tickets;
  int type;          // FL_GGML_Q4_K or FL_GGML_Q6_K
  int nblocks;       // out / 64
  int nsb;           // in / 256
  int slices;
  int slice_sb;      // super-blocks per slice
  int unit_begin;
};

template <int MAXP>
struct Args {
  int nproblems;
  int batch;
  int digit_stride;
  int max_slice_sb;
  int ncta;
  int cta_begin[kMaxCtas + 1];
  Problem p[MAXP];
};

__device__ int g_error;

enum : int { kTileData = 0, kTileEnd = 2 };
enum : int { kFirst = 1, kLast = 2, kNewX = 4 };
struct TileHdr {
  int kind, flags;
  int p, j, b;
  int sb0;   // first super-block of the tile within the slice
  int tsb;   // super-blocks in the tile
  int off;   // byte offset of the first record inside each row slot
};

struct Cursor {
  int p, j, b, u;
};

template <int MAXP>
__device__ __forceinline__ Cursor cursor_at(const Args<MAXP>& a, int u) {
  int p = 0;
  while (p + 1 < a.nproblems && a.p[p + 1].unit_begin <= u) ++p;
  const int local = u - a.p[p].unit_begin;
  Cursor c;
  c.p = p;
  c.j = local / a.p[p].nblocks;
  c.b = local % a.p[p].nblocks;
  c.u = u;
  return c;
}

template <int MAXP>
__device__ __forceinline__ void cursor_next(const Args<MAXP>& a, Cursor& c) {
  ++c.u;
  if (++c.b == a.p[c.p].nblocks) {
    c.b = 0;
    if (++c.j == a.p[c.p].slices) {
      c.j = 0;
      ++c.p;
    }
  }
}

__device__ __forceinline__ int slice_nsb(const Problem& P, int j) { return min(P.slice_sb, P.nsb - j * P.slice_sb); }

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}

__device__ __forceinline__ int byte_u(uint32_t w, int j) { return (int)__byte_perm(w, 0u, 0x4440u | (uint32_t)j); }

// Byte j of w, sign-extended. Uses PTX prmt directly: its selector's top bit
// replicates the selected byte's sign, which __byte_perm does not expose.
__device__ __forceinline__ int byte_s(uint32_t w, int j) {
  const uint32_t sj = 8u | (uint32_t)j;
  const uint32_t sel = (uint32_t)j | (sj << 4) | (sj << 8) | (sj << 12);
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "r"(sel));
  return (int)r;
}

__device__ __forceinline__ uint32_t lds_u32(const uint8_t* p) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ uint4 lds_v4(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(smem_u32(p)));
  return v;
}

// ---------------------------------------------------------------- Q4_K: half (4 sub-blocks) of one super-block
template <int NT>
__device__ __forceinline__ void q4k_half(const uint8_t* rec0, const uint8_t* rec1, int half, const int8_t* const (&dl)[NT],
                                         const int (&dstep)[NT], int colg, const float* inv_scale, const int32_t* gsum,
                                         int gstride, int gi, int t, float (&acc)[NT][2]) {
  const uint4 h0 = lds_v4(rec0);
  const uint4 h1 = lds_v4(rec1);
  const float d0 = half_bits_to_float(h0.x), dm0 = half_bits_to_float(h0.x >> 16);
  const float d1 = half_bits_to_float(h1.x), dm1 = half_bits_to_float(h1.x >> 16);
  const uint32_t S0 = half ? h0.z : h0.y, S1 = half ? h1.z : h1.y;
  const uint32_t sc0 = S0 & 0x3F3F3F3Fu, sc1 = S1 & 0x3F3F3F3Fu;
  // mn_j bytes: low 2 bits from the top of byte j, high 4 bits from nibble j
  const uint32_t M0 = half ? (h0.w >> 16) : (h0.w & 0xFFFFu), M1 = half ? (h1.w >> 16) : (h1.w & 0xFFFFu);
  const uint32_t mn0 = ((S0 >> 6) & 0x03030303u) | (__byte_perm(M0 & 0x0F0Fu, (M0 >> 4) & 0x0F0Fu, 0x5140u) << 2);
  const uint32_t mn1 = ((S1 >> 6) & 0x03030303u) | (__byte_perm(M1 & 0x0F0Fu, (M1 >> 4) & 0x0F0Fu, 0x5140u) << 2);
  uint32_t q0[4], q1[4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = 4 * half + jj;
    q0[jj] = lds_u32(rec0 + 16 + 16 * j + 4 * t);
    q1[jj] = lds_u32(rec1 + 16 + 16 * j + 4 * t);
  }
  int32_t ai[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) ai[nt][0] = ai[nt][1] = ai[nt][2] = ai[nt][3] = 0;
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = 4 * half + jj;
    const uint32_t a0 = q0[jj] & 0x0F0F0F0Fu, a2 = (q0[jj] >> 4) & 0x0F0F0F0Fu;
    const uint32_t a1 = q1[jj] & 0x0F0F0F0Fu, a3 = (q1[jj] >> 4) & 0x0F0F0F0Fu;
    const int s0 = byte_u(sc0, jj), s1 = byte_u(sc1, jj);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint2 bb = *reinterpret_cast<const uint2*>(dl[nt] + dstep[nt] * (colg + 32 * j));
      int32_t C[4] = {0, 0, 0, 0};
      mma_u8s8(C, a0, a1, a2, a3, bb.x, bb.y);
      ai[nt][0] += s0 * C[0];
      ai[nt][1] += s0 * C[1];
      ai[nt][2] += s1 * C[2];
      ai[nt][3] += s1 * C[3];
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int bb = 4 * nt + t;
    const float isc = inv_scale[bb * gstride + gi];
    // sums over the 32-column sub-blocks from the 16-column sums
    const int4 Xa = *reinterpret_cast<const int4*>(gsum + (bb * gstride + gi) * 8);
    const int4 Xb = *reinterpret_cast<const int4*>(gsum + (bb * gstride + gi) * 8 + 4);
    const int32_t X0 = Xa.x + Xa.y, X1 = Xa.z + Xa.w, X2 = Xb.x + Xb.y, X3 = Xb.z + Xb.w;
    const int32_t mx0 = byte_u(mn0, 0) * X0 + byte_u(mn0, 1) * X1 + byte_u(mn0, 2) * X2 + byte_u(mn0, 3) * X3;
    const int32_t mx1 = byte_u(mn1, 0) * X0 + byte_u(mn1, 1) * X1 + byte_u(mn1, 2) * X2 + byte_u(mn1, 3) * X3;
    const float v0 = fmaf(256.f, (float)ai[nt][0], (float)ai[nt][1]);
    const float v1 = fmaf(256.f, (float)ai[nt][2], (float)ai[nt][3]);
    acc[nt][0] = fmaf(isc, fmaf(d0, v0, -dm0 * (float)mx0), acc[nt][0]);
    acc[nt][1] = fmaf(isc, fmaf(d1, v1, -dm1 * (float)mx1), acc[nt][1]);
  }
}

// ---------------------------------------------------------------- Q6_K: half (8 sub-blocks of 16) of one super-block
template <int NT>
__device__ __forceinline__ void q6k_half(const uint8_t* rec0, const uint8_t* rec1, int odd, int half,
                                         const int8_t* const (&dl)[NT], const int (&dstep)[NT], int colg,
                                         const float* inv_scale, const int32_t* gsum, int gstride, int gi, int t,
                                         float (&acc)[NT][2]) {
  const uint8_t* qa0 = rec0 + (odd ? 2 : 0);
  const uint8_t* qa1 = rec1 + (odd ? 2 : 0);
  const uint8_t* sc0p = rec0 + (odd ? 194 : 192);
  const uint8_t* sc1p = rec1 + (odd ? 194 : 192);
  const float d0 = half_bits_to_float(*reinterpret_cast<const uint16_t*>(rec0 + (odd ? 0 : 208)));
  const float d1 = half_bits_to_float(*reinterpret_cast<const uint16_t*>(rec1 + (odd ? 0 : 208)));
  int32_t ai[NT][4], ao[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) ai[nt][0] = ai[nt][1] = ai[nt][2] = ai[nt][3] = ao[nt][0] = ao[nt][1] = 0;
#pragma unroll
  for (int mm = 0; mm < 2; ++mm) {
    const int m = 2 * half + mm;
    const uint8_t* w0 = qa0 + 48 * t + 12 * m;
    const uint8_t* w1 = qa1 + 48 * t + 12 * m;
    const uint32_t A0 = lds_u32(w0), B0 = lds_u32(w0 + 4), C0 = lds_u32(w0 + 8);
    const uint32_t A1 = lds_u32(w1), B1 = lds_u32(w1 + 4), C1 = lds_u32(w1 + 8);
    const uint32_t scw0 = lds_u32(sc0p + 4 * m), scw1 = lds_u32(sc1p + 4 * m);
    uint32_t op0[4], op1[4];
    op0[0] = (A0 & 0x0F0F0F0Fu) | (C0 & 0x30303030u);
    op0[1] = ((A0 >> 4) & 0x0F0F0F0Fu) | ((C0 >> 2) & 0x30303030u);
    op0[2] = (B0 & 0x0F0F0F0Fu) | ((C0 << 4) & 0x30303030u);
    op0[3] = ((B0 >> 4) & 0x0F0F0F0Fu) | ((C0 << 2) & 0x30303030u);
    op1[0] = (A1 & 0x0F0F0F0Fu) | (C1 & 0x30303030u);
    op1[1] = ((A1 >> 4) & 0x0F0F0F0Fu) | ((C1 >> 2) & 0x30303030u);
    op1[2] = (B1 & 0x0F0F0F0Fu) | ((C1 << 4) & 0x30303030u);
    op1[3] = ((B1 >> 4) & 0x0F0F0F0Fu) | ((C1 << 2) & 0x30303030u);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int j = 4 * m + s;  // sub-block of 16 weights
      const int s0 = byte_s(scw0, s), s1 = byte_s(scw1, s);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(dl[nt] + dstep[nt] * (colg + 16 * j));
        int32_t C[4] = {0, 0, 0, 0};
        mma_u8s8_k16(C, op0[s], op1[s], b0);
        ai[nt][0] += s0 * C[0];
        ai[nt][1] += s0 * C[1];
        ai[nt][2] += s1 * C[2];
        ai[nt][3] += s1 * C[3];
        const int32_t X = gsum[((4 * nt + t) * gstride + gi) * 8 + (j & 7)];
        ao[nt][0] += s0 * X;
        ao[nt][1] += s1 * X;
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float isc = inv_scale[(4 * nt + t) * gstride + gi];
    const float v0 = fmaf(256.f, (float)ai[nt][0], fmaf(-32.f, (float)ao[nt][0], (float)ai[nt][1]));
    const float v1 = fmaf(256.f, (float)ai[nt][2], fmaf(-32.f, (float)ao[nt][1], (float)ai[nt][3]));
    acc[nt][0] = fmaf(isc * d0, v0, acc[nt][0]);
    acc[nt][1] = fmaf(isc * d1, v1, acc[nt][1]);
  }
}

template <int MAXP, int NT>
__global__ void __launch_bounds__(kThreads, 1) kquant_gemv_kernel(const __grid_constant__ Args<MAXP> a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ TileHdr hdr[kStages];
  __shared__ __align__(16) uint8_t zeros[160];
  __shared__ int s_ticket;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u_begin = a.cta_begin[blockIdx.x], u_end = a.cta_begin[blockIdx.x + 1];
  if (u_begin >= u_end) return;
  uint8_t* stages = smem;
  int8_t* digits = reinterpret_cast<int8_t*>(smem + kStages * kStageBytes);
  const int ndrows = 2 * a.batch;
  const int max_groups = 2 * a.max_slice_sb;
  float* inv_scale = reinterpret_cast<float*>(smem + kStages * kStageBytes + (size_t)ndrows * a.digit_stride);
  int32_t* gsum = reinterpret_cast<int32_t*>(inv_scale + 4 * NT * max_groups);
  float* xfer = reinterpret_cast<float*>(gsum + 4 * NT * max_groups * 8);  // [4 mt][3][NT][64]

  if (threadIdx.x < 40) reinterpret_cast<uint32_t*>(zeros)[threadIdx.x] = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer warp: all lanes issue row copies
    int s = 0;
    uint32_t phase = 0, issued = 0;
    int last_p = -1, last_j = -1;
    Cursor c = cursor_at(a, u_begin);
    for (; c.u < u_end; cursor_next(a, c)) {
      const Problem& P = a.p[c.p];
      const bool q4 = P.type == FL_GGML_Q4_K;
      const int rec = q4 ? 144 : 210, tsbm = q4 ? kQ4Tsb : kQ6Tsb, slot = q4 ? kQ4Slot : kQ6Slot;
      const int sb0s = c.j * P.slice_sb, nsbs = slice_nsb(P, c.j);
      for (int t0 = 0; t0 < nsbs; t0 += tsbm) {
        const int tsb = min(tsbm, nsbs - t0);
        if (issued >= (uint32_t)kStages) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait(&empty_bar[s], phase ^ 1u);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            if (lane == 0) atomicExch(&g_error, 1);
            return;
          }
        }
        const size_t start_off = (size_t)rec * (sb0s + t0);
        const size_t a_off = start_off & ~(size_t)15;
        const size_t e_off = (start_off + (size_t)rec * tsb + 15) & ~(size_t)15;
        const uint32_t row_bytes = (uint32_t)(e_off - a_off);
        uint8_t* st = stages + s * kStageBytes;
        if (lane == 0) {
          TileHdr& h = hdr[s];
          h.kind = kTileData;
          int fl = (t0 == 0 ? kFirst : 0) | (t0 + tsb >= nsbs ? kLast : 0);
          if (t0 == 0 && (c.p != last_p || c.j != last_j)) fl |= kNewX;
          h.flags = fl;
          h.p = c.p;
          h.j = c.j;
          h.b = c.b;
          h.sb0 = t0;
          h.tsb = tsb;
          h.off = (int)(start_off - a_off);
          mbar_expect_tx(&full_bar[s], row_bytes * 64u);
        }
        if (t0 == 0) {
          last_p = c.p;
          last_j = c.j;
        }
        __syncwarp();
        for (int r = lane; r < 64; r += 32) {
          const uint8_t* src = P.blocks + (size_t)(64 * c.b + r) * P.nsb * rec + a_off;
          bulk_g2s(st + slot * r, src, row_bytes, &full_bar[s]);
        }
        ++issued;
        if (++s == kStages) {
          s = 0;
          phase ^= 1u;
        }
      }
    }
    if (issued >= (uint32_t)kStages) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty_bar[s], phase ^ 1u);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return;
    }
    if (lane == 0) {
      hdr[s].kind = kTileEnd;
      mbar_arrive(&full_bar[s]);
    }
    return;
  }

  // -------------------------------------------------------------- consumer warps
  const int mt = warp & 3, sq = warp >> 2;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * mt + g;
  const int8_t* dl_perm[NT];
  const int8_t* dl_nat[NT];
  int dstep[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int row = 8 * nt + g;
    const bool live = row < ndrows;
    dl_perm[nt] = live ? digits + (size_t)row * a.digit_stride + 8 * t : reinterpret_cast<const int8_t*>(zeros) + 8 * t;
    dl_nat[nt] = live ? digits + (size_t)row * a.digit_stride + 4 * t : reinterpret_cast<const int8_t*>(zeros) + 4 * t;
    dstep[nt] = live ? 1 : 0;
  }
  float acc[NT][2];
  int gstride = 2;
  int s = 0;
  uint32_t phase = 0;
  for (;;) {
    if (!mbar_wait(&full_bar[s], phase)) {
      if (lane == 0) atomicExch(&g_error, 2);
      return;
    }
    const TileHdr h = hdr[s];
    if (h.kind == kTileEnd) break;
    const Problem& P = a.p[h.p];
    const bool q4 = P.type == FL_GGML_Q4_K;
    if (h.flags & kNewX) {
      named_bar(1, kConsumers);
      gstride = 2 * slice_nsb(P, h.j);
      XDigitView v;
      v.digits = digits;
      v.inv_scale = inv_scale;
      v.gsum = gsum;
      v.stride = a.digit_stride;
      v.ngroups = gstride;
      build_x_digits(P.x, P.nsb * 256, a.batch, 4 * NT, 256 * h.j * P.slice_sb, v, 8, threadIdx.x, kConsumers,
                     q4 ? 1 : 0);
      named_bar(1, kConsumers);
    }
    if (h.flags & kFirst) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
    }
    const uint8_t* st = stages + s * kStageBytes;
    const int rec = q4 ? 144 : 210, slot = q4 ? kQ4Slot : kQ6Slot;
    // work items of the tile: (super-block k, half) = 2 tsb halves, item hh = 2 k + half
    for (int hh = sq; hh < 2 * h.tsb; hh += 4) {
      const int k = hh >> 1, half = hh & 1;
      const uint8_t* rec0 = st + slot * r0 + h.off + rec * k;
      const uint8_t* rec1 = rec0 + slot * 8;
      const int sbs = h.sb0 + k;
      const int gi = 2 * sbs + half;
      if (q4)
        q4k_half<NT>(rec0, rec1, half, dl_perm, dstep, 256 * sbs, inv_scale, gsum, gstride, gi, t, acc);
      else
        q6k_half<NT>(rec0, rec1, (h.j * P.slice_sb + sbs) & 1, half, dl_nat, dstep, 256 * sbs, inv_scale, gsum,
                     gstride, gi, t, acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
    if (++s == kStages) {
      s = 0;
      phase ^= 1u;
    }
    if (!(h.flags & kLast)) continue;

    float* xf = xfer + (size_t)mt * 3 * NT * 64;
    if (sq > 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        xf[((sq - 1) * NT + nt) * 64 + lane] = acc[nt][0];
        xf[((sq - 1) * NT + nt) * 64 + 32 + lane] = acc[nt][1];
      }
    }
    named_bar(2 + mt, 128);
    if (sq == 0) {
#pragma unroll
      for (int q = 0; q < 3; ++q)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[nt][0] += xf[(q * NT + nt) * 64 + lane];
          acc[nt][1] += xf[(q * NT + nt) * 64 + 32 + lane];
        }
    }
    named_bar(2 + mt, 128);
    const size_t ystride = (size_t)64 * P.nblocks;
    const int row_base = 64 * h.b + 16 * mt;
    if (P.slices == 1) {
      if (sq == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int bb = 4 * nt + t;
          if (bb < a.batch) {
            float* y0 = P.y + (size_t)bb * ystride + row_base + g;
            y0[0] = acc[nt][0];
            y0[8] = acc[nt][1];
          }
        }
      }
    } else {
      if (sq == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int bb = 4 * nt + t;
          if (bb < a.batch) {
            float* pp = P.partial + (((size_t)h.j * P.nblocks + h.b) * a.batch + bb) * 64 + 16 * mt + g;
            pp[0] = acc[nt][0];
            pp[8] = acc[nt][1];
          }
        }
      }
      __threadfence();
      named_bar(1, kConsumers);
      if (threadIdx.x == 0) s_ticket = (int)atomicAdd(&P.tickets[h.b], 1u);
      named_bar(1, kConsumers);
      if (s_ticket == P.slices - 1) {
        __threadfence();
        for (int e = threadIdx.x; e < a.batch * 64; e += kConsumers) {
          const int bb = e / 64, r = e % 64;
          float sum = 0.f;
          for (int jj = 0; jj < P.slices; ++jj)
            sum += __ldcg(P.partial + (((size_t)jj * P.nblocks + h.b) * a.batch + bb) * 64 + r);
          P.y[(size_t)bb * ystride + 64 * h.b + r] = sum;
        }
        if (threadIdx.x == 0) P.tickets[h.b] = 0u;
      }
      named_bar(1, kConsumers);
    }
  }
}

// ---------------------------------------------------------------- host side

struct Plan {
  int slices, slice_sb;
};

// Dynamic shared memory: stages, activation digits, per (padded batch, 128-column group)
// the inverse scale plus 8 sub-group sums, and the cross-warp transfer of row sums.
static size_t smem_bytes(int batch, int slice_sb) {
  const int nt = (batch + 3) / 4;
  return (size_t)kStages * kStageBytes + (size_t)2 * batch * (256 * slice_sb + 16) +
         (size_t)4 * nt * (2 * slice_sb) * 36 + (size_t)3072 * nt;
}

static int max_sb_fit(int batch) {
  const int nt = (batch + 3) / 4;
  const long avail = (long)kSmemLimit - (long)kStages * kStageBytes - 32L * batch - 3072L * nt;
  return (int)std::max(1L, avail / (512L * batch + 288L * nt));
}

static Plan plan_single(int nblocks, int nsb, int batch, int nsm) {
  Plan pl;
  const int max_sb = max_sb_fit(batch);
  const int s_mem = (nsb + max_sb - 1) / max_sb;
  const int s_fill = (2 * nsm + nblocks - 1) / nblocks;
  int s = std::max(s_mem, std::min(s_fill, std::max(1, nsb / 4)));
  s = std::min(s, nsb);
  pl.slice_sb = (nsb + s - 1) / s;
  pl.slices = (nsb + pl.slice_sb - 1) / pl.slice_sb;
  return pl;
}

static size_t workspace_for(const Plan& pl, int nblocks, int batch) {
  if (pl.slices <= 1) return 0;
  const size_t tickets = ((size_t)nblocks * 4 + 255) / 256 * 256;
  return tickets + (size_t)pl.slices * nblocks * batch * 64 * 4;
}

template <int MAXP>
static void partition(Args<MAXP>& a, int nsm) {
  double total = 0;
  for (int i = 0; i < a.nproblems; ++i)
    total += (double)a.p[i].nblocks * a.p[i].nsb * (a.p[i].type == FL_GGML_Q4_K ? 144 : 210);
  const Problem& L = a.p[a.nproblems - 1];
  const int units = L.unit_begin + L.nblocks * L.slices;
  int ncta = std::max(1, std::min(std::min(nsm, units), kMaxCtas));
  a.ncta = ncta;
  int c = 0;
  a.cta_begin[0] = 0;
  double acc = 0;
  for (int i = 0; i < a.nproblems && c < ncta; ++i) {
    const Problem& P = a.p[i];
    const int nu = P.nblocks * P.slices;
    const double per = (double)P.nsb * (P.type == FL_GGML_Q4_K ? 144 : 210) / P.slices;
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
  const size_t smem = smem_bytes(a.batch, a.max_slice_sb);
  auto kern = kquant_gemv_kernel<MAXP, NT>;
  FL_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                "cudaFuncSetAttribute(kquant_gemv)");
  kern<<<a.ncta, kThreads, smem, st>>>(a);
  FL_CHECK_CUDA(cudaGetLastError(), "launch kquant_gemv");
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

static fl_status check_tensor(const void* blocks, int type, int out, int in, const char* what, int idx) {
  if (type != FL_GGML_Q4_K && type != FL_GGML_Q6_K)
    return fail(FL_ERR_UNSUPPORTED, "%s: tensor %d has GGUF type %d; the fast path implements Q4_K (12) and Q6_K (14)",
                what, idx, type);
  if (!blocks) return fail(FL_ERR_ARG, "%s: tensor %d blocks pointer is NULL", what, idx);
  if (out <= 0 || out % 64 || in <= 0 || in % 256 || (type == FL_GGML_Q6_K && in % 2048))
    return fail(FL_ERR_SHAPE, "%s: tensor %d out=%d in=%d (out %% 64 == 0, in %% 256 == 0, Q6_K in %% 2048 == 0)",
                what, idx, out, in);
  if (!aligned16(blocks)) return fail(FL_ERR_ALIGN, "%s: tensor %d blocks not 16-byte aligned", what, idx);
  return FL_OK;
}

}  // namespace kq
}  // namespace fl

using namespace fl;

extern "C" size_t fl_kquant_bytes(int ggml_type, int out, int in) {
  if (out <= 0 || in <= 0 || in % 256) return 0;
  if (ggml_type == FL_GGML_Q4_K) return (size_t)out * (in / 256) * 144u;
  if (ggml_type == FL_GGML_Q6_K) return (size_t)out * (in / 256) * 210u;
  return 0;
}

extern "C" size_t fl_kquant_workspace_bytes(int ggml_type, int out, int in, int batch) {
  if (ggml_type != FL_GGML_Q4_K && ggml_type != FL_GGML_Q6_K) return 0;
  if (out <= 0 || out % 64 || in <= 0 || in % 256 || batch < 1 || batch > FL_MAX_BATCH) return 0;
  const int nsm = device_sm_count();
  if (nsm <= 0) return 0;
  kq::Plan pl = kq::plan_single(out / 64, in / 256, batch, nsm);
  return kq::workspace_for(pl, out / 64, batch);
}

extern "C" fl_status fl_gemv_kquant(const void* blocks, int ggml_type, int out, int in, const uint16_t* x, int batch,
                                    float* y, void* workspace, size_t workspace_bytes, void* stream) {
  const char* what = "fl_gemv_kquant";
  fl_status st = kq::check_tensor(blocks, ggml_type, out, in, what, 0);
  if (st != FL_OK) return st;
  if (!x || !y) return fail(FL_ERR_ARG, "%s: NULL x/y", what);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  if (!aligned16(x)) return fail(FL_ERR_ALIGN, "%s: x not 16-byte aligned", what);
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  const int nblocks = out / 64, nsb = in / 256;
  kq::Plan pl = kq::plan_single(nblocks, nsb, batch, nsm);
  const size_t need = kq::workspace_for(pl, nblocks, batch);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(FL_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", what, workspace ? workspace_bytes : (size_t)0,
                need);
  if (need > 0 && !aligned16(workspace)) return fail(FL_ERR_ALIGN, "%s: workspace not 16-byte aligned", what);
  static thread_local kq::Args<1> a;
  a.nproblems = 1;
  a.batch = batch;
  a.max_slice_sb = pl.slice_sb;
  a.digit_stride = 256 * pl.slice_sb + 16;
  kq::Problem& P = a.p[0];
  P.blocks = static_cast<const uint8_t*>(blocks);
  P.x = x;
  P.y = y;
  P.type = ggml_type;
  P.nblocks = nblocks;
  P.nsb = nsb;
  P.slices = pl.slices;
  P.slice_sb = pl.slice_sb;
  P.unit_begin = 0;
  if (pl.slices > 1) {
    const size_t tick = ((size_t)nblocks * 4 + 255) / 256 * 256;
    P.tickets = static_cast<uint32_t*>(workspace);
    P.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + tick);
  } else {
    P.tickets = nullptr;
    P.partial = nullptr;
  }
  kq::partition(a, nsm);
  return kq::launch_nt(a, static_cast<cudaStream_t>(stream));
}

extern "C" fl_status fl_gemv_kquant_batched(const fl_kquant_problem* problems, int n, int batch, void* stream) {
  const char* what = "fl_gemv_kquant_batched";
  if (!problems) return fail(FL_ERR_ARG, "%s: problems is NULL", what);
  if (n < 1 || n > FL_MAX_PROBLEMS) return fail(FL_ERR_ARG, "%s: n=%d (1..%d)", what, n, FL_MAX_PROBLEMS);
  if (batch < 1 || batch > FL_MAX_BATCH) return fail(FL_ERR_SHAPE, "%s: batch=%d (1..16)", what, batch);
  static thread_local kq::Args<FL_MAX_PROBLEMS> a;
  a.nproblems = n;
  a.batch = batch;
  int max_sb = 0, unit = 0;
  for (int i = 0; i < n; ++i) {
    const fl_kquant_problem& q = problems[i];
    fl_status st = kq::check_tensor(q.blocks, q.ggml_type, q.out, q.in, what, i);
    if (st != FL_OK) return st;
    if (!q.x || !q.y) return fail(FL_ERR_ARG, "%s: tensor %d NULL x/y", what, i);
    if (!aligned16(q.x)) return fail(FL_ERR_ALIGN, "%s: tensor %d x not 16-byte aligned", what, i);
    const int nsb = q.in / 256;
    if (nsb > kq::max_sb_fit(batch))
      return fail(FL_ERR_SHAPE, "%s: tensor %d in=%d too wide for batch %d in one launch (in <= %d)", what, i, q.in,
                  batch, 256 * kq::max_sb_fit(batch));
    kq::Problem& P = a.p[i];
    P.blocks = static_cast<const uint8_t*>(q.blocks);
    P.x = q.x;
    P.y = q.y;
    P.partial = nullptr;
    P.tickets = nullptr;
    P.type = q.ggml_type;
    P.nblocks = q.out / 64;
    P.nsb = nsb;
    P.slices = 1;
    P.slice_sb = nsb;
    P.unit_begin = unit;
    unit += P.nblocks;
    max_sb = std::max(max_sb, nsb);
  }
  a.max_slice_sb = max_sb;
  a.digit_stride = 256 * max_sb + 16;
  const int nsm = device_sm_count();
  if (nsm <= 0) return fail(FL_ERR_CUDA, "%s: no CUDA device", what);
  kq::partition(a, nsm);
  return kq::launch_nt(a, static_cast<cudaStream_t>(stream));
}
